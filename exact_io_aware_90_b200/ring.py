"""Ring (context-parallel) attention forward: one long sequence split over the ranks of a process group.

Rank r of W holds positions [r·S, (r+1)·S) of q, k and v ([S, H, d] each, one sequence).  The K/V
shards travel once around the ring — rank r sends the shard in hand to rank r+1 and receives the
next one from rank r−1 (NCCL send/recv into local buffers, overlapped with the block computed on the
shard in hand).  At step t rank r holds the shard of rank s = (r − t) mod W and attends its queries
to it with the library's forward kernel — the causal diagonal block when s = r, every key when s < r,
nothing when s > r under the causal mask — then folds the block's (O, LSE) into its running result
with the library's merge kernel (FlashAttention 与算子融合, 工程实践 "与 CP 配合": ring attention for
very long sequences with FlashAttention as the compute core; the merge is the block-merge rule of the
same page, "FlashAttention 的两个关键").  Forward only.

The per-rank state (``RingAttention``) is separate from the transport (``ring_attention_forward``),
so the same per-step code runs under NCCL, under another backend, or with the ranks of a ring laid
side by side in one process.
"""

from __future__ import annotations

import math
from typing import Callable, Optional, Tuple

from . import attention_forward, attention_merge


def ring_block(rank: int, step: int, world: int, causal: bool) -> Tuple[int, Optional[str]]:
    """(source rank, kind) of the K/V shard rank `rank` holds at step `step`: kind "causal" (its own,
    diagonal block), "full", or None (a later shard under the causal mask: nothing to compute)."""
    src = (rank - step) % world
    if src == rank:
        return src, "causal" if causal else "full"
    if causal and src > rank:
        return src, None
    return src, "full"


def _default_block(q, k, v, causal, scale, out, lse):
    attention_forward(q, k, v, causal=causal, scale=scale, out=out, lse=lse)


def _default_merge(acc_o, acc_lse, part_o, part_lse, out, first):
    attention_merge(acc_o, acc_lse, part_o, part_lse, out=out, first=first)


class RingAttention:
    """Running result of one rank.  Call ``consume(step, k, v)`` with the shard held at each step
    0 … world−1 (in order), then ``result()`` → (O [S, H, d] in q's dtype, LSE [S, H] fp32).

    ``block_fn(q, k, v, causal, scale, out, lse)`` computes one block and ``merge_fn(acc_o, acc_lse,
    part_o, part_lse, out, first)`` folds it in; both default to the library's kernels.
    """

    def __init__(self, q, rank: int, world: int, causal: bool, scale: Optional[float] = None,
                 block_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
        import torch
        S, H, d = q.shape
        self.q, self.rank, self.world, self.causal = q, rank, world, causal
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        self.block_fn = block_fn or _default_block
        self.merge_fn = merge_fn or _default_merge
        steps = [t for t in range(world) if ring_block(rank, t, world, causal)[1] is not None]
        self.last = steps[-1]
        self.n_parts = len(steps)
        self.done = 0
        self.out = torch.empty_like(q)
        self.lse = torch.empty((S, H), dtype=torch.float32, device=q.device)  # the running LSE, then the result
        if self.n_parts > 1:
            self.acc_o = torch.empty((S, H, d), dtype=torch.float32, device=q.device)
            self.part_o = torch.empty_like(q)
            self.part_lse = torch.empty((S, H), dtype=torch.float32, device=q.device)

    def consume(self, step: int, k, v) -> None:
        _, kind = ring_block(self.rank, step, self.world, self.causal)
        if kind is None:
            return
        causal = kind == "causal"
        if self.n_parts == 1:  # one block: it is the result
            self.block_fn(self.q, k, v, causal, self.scale, self.out, self.lse)
        else:
            self.block_fn(self.q, k, v, causal, self.scale, self.part_o, self.part_lse)
            self.merge_fn(self.acc_o, self.lse, self.part_o, self.part_lse,
                          self.out if step == self.last else None, self.done == 0)
        self.done += 1

    def result(self):
        if self.done != self.n_parts:
            raise RuntimeError("not every step's shard has been consumed")
        return self.out, self.lse


def ring_attention_forward(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None,
                           block_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """O and LSE of this rank's queries; q, k, v are this rank's contiguous shard [S, H, d] of one
    sequence of W·S tokens, W the size of ``group`` (the default process group when None)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    peer = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    ra = RingAttention(q, rank, world, causal, scale, block_fn, merge_fn)
    # received shards alternate between two buffers, so the caller's k and v are only ever sent
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    cur_k, cur_v = k, v
    for t in range(world):
        reqs = []
        if t < world - 1:  # pass the shard in hand on while computing with it
            rk, rv = bufs[t % 2]
            ops = [dist.P2POp(dist.isend, cur_k, nxt, group), dist.P2POp(dist.isend, cur_v, nxt, group),
                   dist.P2POp(dist.irecv, rk, prv, group), dist.P2POp(dist.irecv, rv, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
        ra.consume(t, cur_k, cur_v)
        for r in reqs:
            r.wait()
        if t < world - 1:
            cur_k, cur_v = bufs[t % 2]
    return ra.result()
