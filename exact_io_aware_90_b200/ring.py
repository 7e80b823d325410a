"""Ring (context-parallel) attention forward: one long sequence split over the ranks of a process group.

Rank r of W holds positions [r·S, (r+1)·S) of q, k and v ([S, H, d] each, one sequence).  The K/V
shards travel once around the ring — rank r sends the shard in hand to rank r+1 and receives the
next one from rank r−1 (NCCL send/recv into local buffers, overlapped with the block computed on the
shard in hand).  At step t rank r holds the shard of rank s = (r − t) mod W and attends its queries
to it with the library's forward kernel — the causal diagonal block when s = r, every key when s < r,
nothing when s > r under the causal mask — then folds the block's (O, LSE) into its running result
with the library's merge kernel (FlashAttention 与算子融合, 工程实践 "与 CP 配合": ring attention for
very long sequences with FlashAttention as the compute core; the merge is the block-merge rule of the
same page, "FlashAttention 的两个关键").

The backward runs the same ring.  A block's gradients come from the library's backward kernel given
the global O and LSE of the rank's queries (P recomputed from the global LSE, D from the global O):
its dQ part adds into the rank's fp32 dQ accumulator (the kernel's own reduce-add), its dK and dV
parts add (fa_accumulate) into fp32 accumulators that travel with the key/value shard and are home
after one more step.

The per-rank state (``RingAttention``) is separate from the transport (``ring_attention_forward``),
so the same per-step code runs under NCCL, under another backend, or with the ranks of a ring laid
side by side in one process.

Shard layouts (``layout``): "contiguous" as above, or "zigzag" for a balanced causal ring — the
sequence is cut into 2W equal chunks and rank r holds chunks r and 2W − 1 − r (one from each end,
concatenated in that order).  A block is then a pair of chunks (the rank's query chunk, the held
shard's key chunk): the causal diagonal when they are the same chunk, full when the key chunk comes
first, skipped when it comes later.  Every rank computes the same number of full blocks per step
(two), where with contiguous shards rank W − 1 computes W blocks and rank 0 one.
``zigzag_shard`` / ``zigzag_unshard`` convert between a whole sequence and the ranks' shards.
"""

from __future__ import annotations

import math
from typing import Callable, Optional, Tuple

from . import FA_OK, FAError, attention_forward, attention_merge, dtype_code, lib


def zigzag_chunks(rank: int, world: int) -> Tuple[int, int]:
    """Global chunk indices (of 2·world) held by `rank` in the zigzag layout, in shard order."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x, rank: int, world: int):
    """Rank `rank`'s zigzag shard [2C, ...] of a whole sequence x [L, ...] (L = 2·world·C)."""
    import torch
    C = x.shape[0] // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([x[a * C:(a + 1) * C], x[b * C:(b + 1) * C]]).contiguous()


def zigzag_unshard(shards):
    """The whole sequence from the ranks' zigzag shards (the inverse of ``zigzag_shard``)."""
    import torch
    world = len(shards)
    C = shards[0].shape[0] // 2
    chunks = [None] * (2 * world)
    for r, sh in enumerate(shards):
        a, b = zigzag_chunks(r, world)
        chunks[a], chunks[b] = sh[:C], sh[C:]
    return torch.cat(chunks)


def ring_blocks(rank: int, step: int, world: int, causal: bool, layout: str = "contiguous"):
    """The blocks rank `rank` computes at step `step` on the shard of rank (rank − step) mod world:
    a list of (query part, key part, kind) with kind "causal" (a diagonal block) or "full"; parts index
    the halves of a zigzag shard, or are 0 (the whole shard) in the contiguous layout."""
    if layout == "contiguous":
        _, kind = ring_block(rank, step, world, causal)
        return [] if kind is None else [(0, 0, kind)]
    if layout != "zigzag":
        raise ValueError("layout must be 'contiguous' or 'zigzag'")
    src = (rank - step) % world
    out = []
    for qi, qc in enumerate(zigzag_chunks(rank, world)):
        for ki, kc in enumerate(zigzag_chunks(src, world)):
            if causal and kc > qc:
                continue
            out.append((qi, ki, "causal" if causal and kc == qc else "full"))
    return out


def _part(x, i: int, nparts: int):
    """Part i of nparts equal row ranges of x (a contiguous view)."""
    n = x.shape[0] // nparts
    return x[i * n:(i + 1) * n]


def ring_block(rank: int, step: int, world: int, causal: bool) -> Tuple[int, Optional[str]]:
    """(source rank, kind) of the K/V shard rank `rank` holds at step `step`: kind "causal" (its own,
    diagonal block), "full", or None (a later shard under the causal mask: nothing to compute)."""
    src = (rank - step) % world
    if src == rank:
        return src, "causal" if causal else "full"
    if causal and src > rank:
        return src, None
    return src, "full"


class _Staged:
    """Completion of a host-staged exchange: waits for the CPU transfers, then copies what was received
    into the device tensors (on the current stream)."""

    def __init__(self, reqs, pairs):
        self.reqs, self.pairs = reqs, pairs

    def wait(self):
        for r in self.reqs:
            r.wait()
        for dst, src in self.pairs:
            dst.copy_(src)


def _exchange(sends, recvs, nxt, prv, group):
    """Send ``sends`` to rank ``nxt`` and receive ``recvs`` from rank ``prv`` (tensors of this rank's
    device) → objects with ``wait()``.  NCCL moves device memory directly.  A backend that moves host
    memory only (gloo) gets host copies: the sends are copied out first (which waits for the kernels
    that wrote them), the receives land in host buffers and are copied in by ``wait()``."""
    import torch.distributed as dist
    on_device = any(t.is_cuda for t in list(sends) + list(recvs))
    if not on_device or dist.get_backend(group) == "nccl":
        ops = [dist.P2POp(dist.isend, t, nxt, group) for t in sends] + \
              [dist.P2POp(dist.irecv, t, prv, group) for t in recvs]
        return dist.batch_isend_irecv(ops)
    host_s = [t.cpu() for t in sends]
    host_r = [_host_like(t) for t in recvs]
    ops = [dist.P2POp(dist.isend, t, nxt, group) for t in host_s] + \
          [dist.P2POp(dist.irecv, t, prv, group) for t in host_r]
    return [_Staged(dist.batch_isend_irecv(ops), list(zip(recvs, host_r)))]


def _host_like(t):
    import torch
    return torch.empty(t.shape, dtype=t.dtype, device="cpu")


def _default_block(q, k, v, causal, scale, out, lse):
    attention_forward(q, k, v, causal=causal, scale=scale, out=out, lse=lse)


def _default_merge(acc_o, acc_lse, part_o, part_lse, out, first):
    attention_merge(acc_o, acc_lse, part_o, part_lse, out=out, first=first)


class RingAttention:
    """Running result of one rank.  Call ``consume(step, k, v)`` with the shard held at each step
    0 … world−1 (in order), then ``result()`` → (O [S, H, d] in q's dtype, LSE [S, H] fp32).

    ``block_fn(q, k, v, causal, scale, out, lse)`` computes one block and ``merge_fn(acc_o, acc_lse,
    part_o, part_lse, out, first)`` folds it in; both default to the library's kernels.  ``layout``:
    "contiguous" or "zigzag" (see the module docstring); each query part keeps its own running result.
    """

    def __init__(self, q, rank: int, world: int, causal: bool, scale: Optional[float] = None,
                 block_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None,
                 layout: str = "contiguous"):
        import torch
        S, H, d = q.shape
        self.q, self.rank, self.world, self.causal, self.layout = q, rank, world, causal, layout
        self.np = 1 if layout == "contiguous" else 2  # query / key parts per shard
        if S % self.np:
            raise ValueError("a zigzag shard holds two equal chunks")
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        self.block_fn = block_fn or _default_block
        self.merge_fn = merge_fn or _default_merge
        # per query part: the blocks that feed it, in ring order (the last writes the output dtype)
        self.feeds = [[(t, ki, kind) for t in range(world) for qi, ki, kind in ring_blocks(rank, t, world, causal,
                                                                                           layout) if qi == p]
                      for p in range(self.np)]
        self.done = [0] * self.np
        self.out = torch.empty_like(q)
        self.lse = torch.empty((S, H), dtype=torch.float32, device=q.device)  # the running LSE, then the result
        if any(len(f) > 1 for f in self.feeds):
            self.acc_o = torch.empty((S, H, d), dtype=torch.float32, device=q.device)
            self.part_o = torch.empty_like(q)
            self.part_lse = torch.empty((S, H), dtype=torch.float32, device=q.device)

    def consume(self, step: int, k, v) -> None:
        n = self.np
        for qi, ki, kind in ring_blocks(self.rank, step, self.world, self.causal, self.layout):
            q, kk, vv = _part(self.q, qi, n), _part(k, ki, n), _part(v, ki, n)
            out, lse = _part(self.out, qi, n), _part(self.lse, qi, n)
            causal = kind == "causal"
            if len(self.feeds[qi]) == 1:  # one block: it is the result
                self.block_fn(q, kk, vv, causal, self.scale, out, lse)
            else:
                po, pl = _part(self.part_o, qi, n), _part(self.part_lse, qi, n)
                self.block_fn(q, kk, vv, causal, self.scale, po, pl)
                last = self.done[qi] == len(self.feeds[qi]) - 1
                self.merge_fn(_part(self.acc_o, qi, n), lse, po, pl, out if last else None, self.done[qi] == 0)
            self.done[qi] += 1

    def result(self):
        if any(dn != len(f) for dn, f in zip(self.done, self.feeds)):
            raise RuntimeError("not every step's shard has been consumed")
        return self.out, self.lse


def ring_attention_forward(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None,
                           block_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None,
                           layout: str = "contiguous"):
    """O and LSE of this rank's queries; q, k, v are this rank's shard [S, H, d] of one sequence of W·S
    tokens (``layout``: contiguous, or zigzag as made by ``zigzag_shard``), W the size of ``group``
    (the default process group when None)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    peer = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    ra = RingAttention(q, rank, world, causal, scale, block_fn, merge_fn, layout)
    # received shards alternate between two buffers, so the caller's k and v are only ever sent
    bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    cur_k, cur_v = k, v
    for t in range(world):
        reqs = []
        if t < world - 1:  # pass the shard in hand on while computing with it
            rk, rv = bufs[t % 2]
            reqs = _exchange([cur_k, cur_v], [rk, rv], nxt, prv, group)
        ra.consume(t, cur_k, cur_v)
        for r in reqs:
            r.wait()
        if t < world - 1:
            cur_k, cur_v = bufs[t % 2]
    return ra.result()


class RingAttentionBackward:
    """One rank's backward state.  Call ``consume(step, k, v, dk_acc, dv_acc)`` with the shard held at
    each step and the fp32 dK/dV accumulators travelling with it (``new_accumulators()`` makes the
    rank's own, consumed at step 0), then ``finish(dk_acc, dv_acc)`` with the accumulators of its own
    shard once they are home → (dq, dk, dv) in q's dtype.  o, lse: the ring forward's result; ``layout``
    as for the forward (each query part of a zigzag shard has its own dQ accumulator)."""

    def __init__(self, q, o, lse, do, rank: int, world: int, causal: bool, scale: Optional[float] = None,
                 layout: str = "contiguous"):
        import torch
        S, H, d = q.shape
        self.q, self.o, self.lse, self.do = q, o, lse, do
        self.rank, self.world, self.causal, self.layout = rank, world, causal, layout
        self.np = 1 if layout == "contiguous" else 2
        if S % self.np:
            raise ValueError("a zigzag shard holds two equal chunks")
        self.S, self.H, self.d = S, H, d
        self.C = S // self.np  # rows of a part
        self.scale = 1.0 / math.sqrt(d) if scale is None else scale
        self.dt = dtype_code(q)
        self.stream = torch.cuda.current_stream(q.device).cuda_stream
        self.ws_bytes = lib.fa_bwd_workspace_bytes(self.C, H, d)
        self.ws = [torch.empty(self.ws_bytes, dtype=torch.uint8, device=q.device) for _ in range(self.np)]
        tmp = torch.empty((self.C, H, d), dtype=q.dtype, device=q.device)
        self.tmp_dk, self.tmp_dv = tmp, torch.empty_like(tmp)
        # per query part: D = rowsum(dO ∘ O) of the global output and a zeroed dQ accumulator
        for i in range(self.np):
            self._check(lib.fa_bwd_preprocess(_part(o, i, self.np).data_ptr(), _part(do, i, self.np).data_ptr(), 1, H,
                                              self.C, d, None, self.C, self.dt, self.ws[i].data_ptr(), self.ws_bytes,
                                              self.stream), "fa_bwd_preprocess")

    @staticmethod
    def _check(st, where):
        if st != FA_OK:
            raise FAError(st, where)

    def new_accumulators(self):
        import torch
        return (torch.empty((self.S, self.H, self.d), dtype=torch.float32, device=self.q.device),
                torch.empty((self.S, self.H, self.d), dtype=torch.float32, device=self.q.device))

    def _acc(self, acc, part, out, first):
        self._check(lib.fa_accumulate(acc.data_ptr(), None if part is None else part.data_ptr(),
                                      None if out is None else out.data_ptr(), acc.numel(), self.dt, int(first),
                                      self.stream), "fa_accumulate")

    def consume(self, step: int, k, v, dk_acc, dv_acc) -> None:
        n, started = self.np, set()
        for qi, ki, kind in ring_blocks(self.rank, step, self.world, self.causal, self.layout):
            self._check(lib.fa_bwd_main(_part(self.q, qi, n).data_ptr(), _part(k, ki, n).data_ptr(),
                                        _part(v, ki, n).data_ptr(), _part(self.lse, qi, n).data_ptr(),
                                        _part(self.do, qi, n).data_ptr(), self.tmp_dk.data_ptr(),
                                        self.tmp_dv.data_ptr(), 1, self.H, self.C, self.d, float(self.scale),
                                        int(kind == "causal"), None, self.C, self.dt, self.ws[qi].data_ptr(),
                                        self.ws_bytes, self.stream), "fa_bwd_main")
            # step 0 is the rank's own shard, whose every key part is computed: the first block on a key
            # part starts the shard's accumulators there
            first = step == 0 and ki not in started
            started.add(ki)
            self._acc(_part(dk_acc, ki, n), self.tmp_dk, None, first)
            self._acc(_part(dv_acc, ki, n), self.tmp_dv, None, first)
        # (a step with no block passes the accumulators on unchanged)

    def finish(self, dk_acc, dv_acc):
        import torch
        dq = torch.empty_like(self.q)
        for i in range(self.np):
            self._check(lib.fa_bwd_postprocess(_part(dq, i, self.np).data_ptr(), 1, self.H, self.C, self.d,
                                               float(self.scale), None, self.C, self.dt, self.ws[i].data_ptr(),
                                               self.ws_bytes, self.stream), "fa_bwd_postprocess")
        dk, dv = torch.empty_like(self.q), torch.empty_like(self.q)
        self._acc(dk_acc, None, dk, False)
        self._acc(dv_acc, None, dv, False)
        return dq, dk, dv


def ring_attention_backward(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None, group=None,
                            state=None, layout: str = "contiguous"):
    """dq, dk, dv of this rank's shards for the ring forward that produced (o, lse) on the same group
    (with the same ``layout``).  ``state`` replaces the rank's RingAttentionBackward (an object with the
    same three methods)."""
    import torch
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    peer = (lambda r: r) if group is None else (lambda r: dist.get_global_rank(group, r))
    nxt, prv = peer((rank + 1) % world), peer((rank - 1) % world)
    rb = state if state is not None else RingAttentionBackward(q, o, lse, do, rank, world, causal, scale, layout)
    if world == 1:
        acc = rb.new_accumulators()
        rb.consume(0, k, v, *acc)
        return rb.finish(*acc)
    kv_bufs = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(min(2, world - 1))]
    acc_bufs = [rb.new_accumulators() for _ in range(2)]
    cur_k, cur_v = k, v
    cur_acc = rb.new_accumulators()
    acc_reqs = []
    for t in range(world):
        kv_reqs = []
        if t < world - 1:  # the next shard's K and V stream in while this block computes
            rk, rv = kv_bufs[t % 2]
            kv_reqs = _exchange([cur_k, cur_v], [rk, rv], nxt, prv, group)
        for r in acc_reqs:  # this shard's accumulators have arrived
            r.wait()
        rb.consume(t, cur_k, cur_v, *cur_acc)
        # the accumulators move on once this rank has added to them (after the last step: home)
        nxt_acc = acc_bufs[t % 2]
        acc_reqs = _exchange([cur_acc[0], cur_acc[1]], [nxt_acc[0], nxt_acc[1]], nxt, prv, group)
        for r in kv_reqs:
            r.wait()
        if t < world - 1:
            cur_k, cur_v = kv_bufs[t % 2]
        # the buffers just sent may be reused two steps on, after the sends completed (waited below)
        sent = cur_acc
        cur_acc = nxt_acc
        acc_bufs[t % 2] = sent
    for r in acc_reqs:
        r.wait()
    return rb.finish(*cur_acc)
