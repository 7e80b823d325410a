"""fp64 CPU oracle for exact attention (forward and backward).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product package.

Parity status of each function (what pins it; see ``tests/test_oracle.py``):
* attention_forward       pinned: the pages' worked examples, closed forms,
                          brute-force blockwise recurrence, invariances.
* attention_backward      pinned: central finite differences, sum invariants,
                          closed form for uniform keys.
* attention_forward_rows  pinned: equals attention_forward on every row.
* attention_fwd_bwd_rows  pinned: equals the full forward/backward restricted
                          to the rows.
* online_blockwise_forward, online_softmax_stats, merge_softmax_stats
                          pinned: the pages' printed numbers.
* decode_forward          pinned: the pages' hand example (last query row),
                          the last row of causal self-attention, brute force.
* split_kv_decode         pinned: equals decode_forward for every chunk size;
                          chunk = 1 reduces to the page's per-element recurrence.
* merge_attention_partials
                          pinned: partials over disjoint key sets (any order, an empty
                          one included) merge to decode_forward over all keys; identity
                          and empty parts; no overflow at log-sum-exps near 1000.
* ring_attention_forward  pinned: equals attention_forward for 1 … 6 ranks, causal and not,
                          in the contiguous and the zigzag layout.
* ring_attention_backward pinned: equals attention_backward for 1 … 6 ranks, causal and not,
                          in both layouts.
* zigzag_chunks, ring_blocks
                          pinned: the zigzag ring covers every visible (query, key) chunk
                          pair exactly once, gives every rank the same causal work, and
                          the contiguous schedule does not.
* philox4x32_10           pinned: the generator's published known-answer vectors.
* dropout_keep_mask       pinned: scalar re-derivation of the element mapping,
                          keep fraction within binomial bounds.
* attention_forward_dropout, attention_backward_dropout
                          pinned: p = 0 equals the plain oracle, unbiased over
                          seeds, finite differences with the mask fixed, the
                          D identity.
"""
from .attention import *  # noqa: F401,F403
from .attention import __all__  # noqa: F401
