"""Host-side checks of ring (context-parallel) attention (no GPU).

* The schedule: which shard each rank holds at each step and which blocks it computes.
* The transport and the per-step bookkeeping over real process groups (gloo, world sizes 2 and 4):
  each rank runs ``ring_attention_forward`` with the block and merge steps done by the fp64 oracle on
  CPU tensors (injected through the driver's ``block_fn`` / ``merge_fn`` arguments, which default to
  the CUDA kernels), and its shard of the result must equal the oracle's attention over the whole
  sequence; the caller's K/V shards must come back untouched.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_schedule(world, causal):
    from exact_io_aware_90_b200.ring import ring_block
    for r in range(world):
        held = [ring_block(r, t, world, causal)[0] for t in range(world)]
        # every shard passes through every rank exactly once, its own first, then r−1, r−2, …
        assert held == [(r - t) % world for t in range(world)]
        computed = {src for t in range(world) for src, kind in [ring_block(r, t, world, causal)] if kind}
        assert computed == (set(range(r + 1)) if causal else set(range(world)))
        kinds = {ring_block(r, t, world, causal)[0]: ring_block(r, t, world, causal)[1] for t in range(world)}
        assert kinds[r] == ("causal" if causal else "full")
        assert all(kinds[s] == "full" for s in range(r))


def _oracle_block(q, k, v, causal, scale, out, lse):
    import oracle
    O, L = oracle.attention_forward(q.double().numpy(), k.double().numpy(), v.double().numpy(), scale, causal)
    out.copy_(torch.from_numpy(O).to(out.dtype))
    lse.copy_(torch.from_numpy(L).to(lse.dtype))


def _oracle_merge(acc_o, acc_lse, part_o, part_lse, out, first):
    import oracle
    if first:
        O, L = part_o.double().numpy(), part_lse.double().numpy()
    else:
        O, L = oracle.merge_attention_partials([(acc_o.double().numpy(), acc_lse.double().numpy()),
                                                (part_o.double().numpy(), part_lse.double().numpy())])
    acc_lse.copy_(torch.from_numpy(L).to(acc_lse.dtype))
    (out if out is not None else acc_o).copy_(torch.from_numpy(O).to((out if out is not None else acc_o).dtype))


def _rank_main(rank, world, port, causal, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_io_aware_90_b200.ring import ring_attention_forward
        L, H, d = 24, 2, 8
        g = np.random.default_rng(7)
        q, k, v = (g.standard_normal((L, H, d)) for _ in range(3))
        S = L // world
        sl = slice(rank * S, (rank + 1) * S)
        qs, ks, vs = (torch.from_numpy(x[sl].copy()).to(torch.float64) for x in (q, k, v))
        k0, v0 = ks.clone(), vs.clone()
        o, lse = ring_attention_forward(qs, ks, vs, causal=causal, scale=0.35, block_fn=_oracle_block,
                                        merge_fn=_oracle_merge)
        O_ref, L_ref = oracle.attention_forward(q, k, v, 0.35, causal)
        err = max(float(np.abs(o.numpy() - O_ref[sl]).max()), float(np.abs(lse.numpy() - L_ref[sl]).max()))
        untouched = bool(torch.equal(ks, k0) and torch.equal(vs, v0))
        dist.barrier()
        out_q.put((rank, err, untouched))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_gloo(world, causal):
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, untouched in got:
        assert err < 1e-5, (rank, err)  # the running O and LSE are fp32 buffers, as on the GPU
        assert untouched, rank


class _OracleBackwardState:
    """The per-rank backward steps done by the fp64 oracle on CPU tensors (the same blocks as the
    kernels: P from the global LSE, D from the global O)."""

    def __init__(self, q, o, lse, do, rank, world, causal, scale, layout="contiguous"):
        self.q, self.o, self.lse, self.do = (x.double().numpy() for x in (q, o, lse, do))
        self.rank, self.world, self.causal, self.scale, self.layout = rank, world, causal, scale, layout
        self.np = 1 if layout == "contiguous" else 2
        self.D = (self.do * self.o).sum(axis=-1)
        self.dq = np.zeros_like(self.q)

    def new_accumulators(self):
        return torch.zeros(self.q.shape, dtype=torch.float32), torch.zeros(self.q.shape, dtype=torch.float32)

    def consume(self, step, k, v, dk_acc, dv_acc):
        from exact_io_aware_90_b200.ring import ring_blocks
        K, V = k.double().numpy(), v.double().numpy()
        C = self.q.shape[0] // self.np
        for qi, ki, kind in ring_blocks(self.rank, step, self.world, self.causal, self.layout):
            rq, rk = slice(qi * C, (qi + 1) * C), slice(ki * C, (ki + 1) * C)
            for h in range(self.q.shape[1]):
                Q, Kp, Vp, dO = self.q[rq, h], K[rk, h], V[rk, h], self.do[rq, h]
                P = np.exp((Q @ Kp.T) * self.scale - self.lse[rq, h][:, None])
                if kind == "causal":
                    P[np.triu_indices(C, k=1)] = 0.0
                dS = P * (dO @ Vp.T - self.D[rq, h][:, None])
                self.dq[rq, h] += self.scale * (dS @ Kp)
                dk_acc[rk, h] += torch.from_numpy(self.scale * (dS.T @ Q)).float()
                dv_acc[rk, h] += torch.from_numpy(P.T @ dO).float()

    def finish(self, dk_acc, dv_acc):
        return torch.from_numpy(self.dq), dk_acc.double(), dv_acc.double()


def _rank_main_bwd(rank, world, port, causal, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_io_aware_90_b200.ring import ring_attention_backward
        L, H, d = 24, 2, 8
        g = np.random.default_rng(8)
        q, k, v, do = (g.standard_normal((L, H, d)) for _ in range(4))
        O, LSE = oracle.attention_forward(q, k, v, 0.35, causal)
        S = L // world
        sl = slice(rank * S, (rank + 1) * S)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[sl]))
        state = _OracleBackwardState(t(q), t(O), t(LSE), t(do), rank, world, causal, 0.35)
        ks, vs = t(k), t(v)
        dq, dk, dv = ring_attention_backward(t(q), ks, vs, t(O), t(LSE), t(do), causal=causal, state=state)
        ref = oracle.attention_backward(q, k, v, do, 0.35, causal)
        err = max(float(np.abs(a.numpy() - b[sl]).max()) for a, b in zip((dq, dk, dv), ref))
        dist.barrier()
        out_q.put((rank, err, bool(torch.equal(ks, t(k)) and torch.equal(vs, t(v)))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_backward_gloo(world, causal):
    """The backward ring's transport over gloo: K/V shards and their travelling dK/dV accumulators
    reach every rank in order and come home; every rank's gradients equal the oracle's over the whole
    sequence (to the fp32 accumulators)."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_bwd, args=(r, world, port, causal, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, untouched in got:
        assert err < 1e-5, (rank, err)
        assert untouched, rank


def _rank_main_single(port, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_io_aware_90_b200.ring import ring_attention_backward, ring_attention_forward
        g = np.random.default_rng(9)
        q, k, v, do = (g.standard_normal((16, 2, 8)) for _ in range(4))
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        o, lse = ring_attention_forward(t(q), t(k), t(v), causal=True, scale=0.3, block_fn=_oracle_block,
                                        merge_fn=_oracle_merge)
        O_ref, L_ref = oracle.attention_forward(q, k, v, 0.3, True)
        state = _OracleBackwardState(t(q), o.double(), lse.double(), t(do), 0, 1, True, 0.3)
        grads = ring_attention_backward(t(q), t(k), t(v), o, lse, t(do), causal=True, state=state)
        ref = oracle.attention_backward(q, k, v, do, 0.3, True)
        err = max([float(np.abs(o.numpy() - O_ref).max()), float(np.abs(lse.numpy() - L_ref).max())] +
                  [float(np.abs(a.numpy() - b).max()) for a, b in zip(grads, ref)])
        out_q.put(err)
    finally:
        dist.destroy_process_group()


def test_ring_single_rank_gloo():
    """A ring of one rank: no exchange, the whole sequence is the rank's own (causal) block."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_rank_main_single, args=(_free_port(), q))
    p.start()
    err = q.get(timeout=120)
    p.join(timeout=60)
    assert p.exitcode == 0 and err < 1e-5, err


# ----------------------------------------------------------------------------- load-balanced (zigzag) layout


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_schedule(world, causal):
    """Every visible (query chunk, key chunk) pair is computed exactly once over the ring, with the
    diagonal pairs causal; under the causal mask every rank computes two full blocks per step (the
    diagonal ones of step 0 counting half each); the shards cut a sequence and put it back."""
    from exact_io_aware_90_b200.ring import ring_blocks, zigzag_chunks, zigzag_shard, zigzag_unshard
    seen = {}
    for r in range(world):
        work = []
        for t in range(world):
            src = (r - t) % world
            w_t = 0.0
            for qi, ki, kind in ring_blocks(r, t, world, causal, "zigzag"):
                qc, kc = zigzag_chunks(r, world)[qi], zigzag_chunks(src, world)[ki]
                seen[(qc, kc)] = seen.get((qc, kc), 0) + 1
                assert kind == ("causal" if causal and qc == kc else "full")
                w_t += 0.5 if kind == "causal" else 1.0
            work.append(w_t)
        if causal:
            assert work == [2.0] * world
    want = {(a, b) for a in range(2 * world) for b in range(2 * world) if not causal or b <= a}
    assert set(seen) == want and all(n == 1 for n in seen.values())
    x = torch.arange(2 * world * 3 * 2, dtype=torch.float32).reshape(2 * world * 3, 2)
    shards = [zigzag_shard(x, r, world) for r in range(world)]
    assert torch.equal(zigzag_unshard(shards), x)
    assert torch.equal(shards[0][:3], x[:3]) and torch.equal(shards[0][3:], x[-3:])


def _rank_main_zigzag(rank, world, port, causal, out_q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from exact_io_aware_90_b200.ring import ring_attention_backward, ring_attention_forward, zigzag_shard
        L, H, d = 2 * world * 5, 2, 8
        g = np.random.default_rng(17)
        q, k, v, do = (torch.from_numpy(g.standard_normal((L, H, d))) for _ in range(4))
        sh = lambda x: zigzag_shard(x, rank, world)
        ks, vs = sh(k), sh(v)
        k0, v0 = ks.clone(), vs.clone()
        o, lse = ring_attention_forward(sh(q), ks, vs, causal=causal, scale=0.35, block_fn=_oracle_block,
                                        merge_fn=_oracle_merge, layout="zigzag")
        O_ref, L_ref = oracle.attention_forward(q.numpy(), k.numpy(), v.numpy(), 0.35, causal)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
        err = max(float(np.abs(o.numpy() - sh(t(O_ref)).numpy()).max()),
                  float(np.abs(lse.numpy() - sh(t(L_ref)).numpy()).max()))
        state = _OracleBackwardState(sh(q), sh(t(O_ref)), sh(t(L_ref)), sh(do), rank, world, causal, 0.35, "zigzag")
        grads = ring_attention_backward(sh(q), ks, vs, sh(t(O_ref)), sh(t(L_ref)), sh(do), causal=causal,
                                        state=state, layout="zigzag")
        ref = oracle.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), 0.35, causal)
        gerr = max(float(np.abs(a.numpy() - sh(t(b)).numpy()).max()) for a, b in zip(grads, ref))
        untouched = bool(torch.equal(ks, k0) and torch.equal(vs, v0))
        dist.barrier()
        out_q.put((rank, err, gerr, untouched))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_ring_gloo(world, causal):
    """The zigzag ring's forward and backward over gloo (oracle steps injected): every rank's shard of
    O, LSE and the gradients equals the oracle's over the whole sequence, cut the same way."""
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main_zigzag, args=(r, world, port, causal, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, gerr, untouched in got:
        assert err < 1e-5 and gerr < 1e-5, (rank, err, gerr)
        assert untouched, rank
