"""GPU parity of the partial-result merge kernel and of ring (context-parallel) attention, through the C ABI.

Every run here has one GPU, so the ring's ranks are laid side by side in one process: each emulated rank
runs exactly the per-step code it runs under NCCL (``RingAttention.consume`` with the library's
forward and merge kernels), and the K/V shards move between steps by rotation instead of send/recv
(the transport itself is covered by the gloo tests of ``test_ring_host.py``).  No kernel waits on
another rank's kernel.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _gpu import LSE_TOL, O_TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    return m


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("d", [64, 128])
def test_merge_kernel(fa, dtype, d):
    """Three partials merged one at a time (the first with first=1, the last into `out`) against the
    oracle's merge of the same (rounded) partials; rows where some or all parts are empty (LSE = −∞)
    and log-sum-exps far from 0 included."""
    T, H = 301, 3
    g = torch.Generator().manual_seed(d)
    tdt = workloads.TORCH_DTYPES[dtype]
    parts = []
    for i in range(3):
        o = torch.randn(T, H, d, generator=g).to(tdt)
        lse = torch.randn(T, H, generator=g) * 3.0 + 20.0 * (i - 1)  # −20 … 20 around the part index
        parts.append((o, lse))
    parts[1][1][:40] = -float("inf")        # part 1 empty on the first rows
    parts[0][1][10:20] = -float("inf")      # all three empty on rows 10–19
    parts[2][1][10:20] = -float("inf")
    parts[0][0][10:20] = 0
    parts[2][1][50:60] += 60.0              # a dominant part
    dev = torch.device("cuda")
    acc_o = torch.empty(T, H, d, dtype=torch.float32, device=dev)
    acc_l = torch.empty(T, H, dtype=torch.float32, device=dev)
    out = torch.empty(T, H, d, dtype=tdt, device=dev)
    for i, (o, l) in enumerate(parts):
        fa.attention_merge(acc_o, acc_l, o.to(dev), l.to(dev), out=out if i == 2 else None, first=(i == 0))
    O_ref, L_ref = oracle.merge_attention_partials([(o, l) for o, l in parts])
    got_l = f64(acc_l)
    assert np.array_equal(np.isneginf(got_l), np.isneginf(L_ref))
    fin = ~np.isneginf(L_ref)
    assert np.max(np.abs(got_l[fin] - L_ref[fin])) <= 1e-5 * 80.0
    assert np.all(f64(out)[~fin] == 0.0)
    assert max_abs(f64(out), O_ref) <= O_TOL
    # the fp32 running result after two parts (no output conversion): tighter
    fa.attention_merge(acc_o, acc_l, parts[0][0].to(dev), parts[0][1].to(dev), first=True)
    fa.attention_merge(acc_o, acc_l, parts[1][0].to(dev), parts[1][1].to(dev))
    O2, L2 = oracle.merge_attention_partials(parts[:2])
    assert max_abs(f64(acc_o), O2) <= 1e-5 * max(1.0, float(np.abs(O2).max()))


def _ring_local(fa, q, k, v, world, causal, scale):
    from exact_io_aware_90_b200.ring import RingAttention
    L = q.shape[0]
    S = L // world
    shard = lambda x, r: x[r * S:(r + 1) * S]
    ras = [RingAttention(shard(q, r), r, world, causal, scale) for r in range(world)]
    held = [(shard(k, r), shard(v, r)) for r in range(world)]
    for t in range(world):
        for r in range(world):
            ras[r].consume(t, *held[r])
        held = [held[(r - 1) % world] for r in range(world)]  # rank r receives what rank r−1 held
    outs = [ra.result() for ra in ras]
    return torch.cat([o for o, _ in outs]), torch.cat([l for _, l in outs])


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("S", [128, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_emulated(fa, world, S, d, causal):
    inp = workloads.random_inputs(2, d, "bf16", seed=900 + world + S + d + int(causal), B=1, N=world * S,
                                  causal=causal, backward=False)
    dev = torch.device("cuda")
    o, lse = _ring_local(fa, inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), world, causal, inp.scale)
    O_ref, L_ref = oracle.attention_forward(inp.q, inp.k, inp.v, inp.scale, causal)
    assert max_abs(f64(o), O_ref) <= O_TOL
    assert max_abs(f64(lse), L_ref) <= LSE_TOL


def test_ring_attention_long_sampled(fa):
    """8 ranks × 2048 tokens (a 16k causal sequence), d = 128: 64 sampled rows against the oracle's
    row-restricted forward, and the ring result against the single-call forward of the whole sequence."""
    world, S = 8, 2048
    inp = workloads.random_inputs(4, 128, "bf16", seed=4242, B=1, N=world * S, causal=True, backward=False)
    dev = torch.device("cuda")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    o, lse = _ring_local(fa, q, k, v, world, True, inp.scale)
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(world * S, 56, replace=False),
                                     [0, S - 1, S, 2 * S, 5 * S + 7, world * S - 1]]))
    O_r, L_r = oracle.attention_forward_rows(inp.q, inp.k, inp.v, rows, inp.scale, True)
    assert max_abs(f64(o)[rows], O_r) <= O_TOL
    assert max_abs(f64(lse)[rows], L_r) <= LSE_TOL
    o1, l1 = fa.attention_forward(q, k, v, causal=True, scale=inp.scale)
    assert max_abs(f64(o), f64(o1)) <= O_TOL and max_abs(f64(lse), f64(l1)) <= LSE_TOL


def _ring_local_bwd(q, k, v, o, lse, do, world, causal, scale):
    from exact_io_aware_90_b200.ring import RingAttentionBackward
    S = q.shape[0] // world
    sh = lambda x, r: x[r * S:(r + 1) * S]
    rbs = [RingAttentionBackward(sh(q, r), sh(o, r), sh(lse, r), sh(do, r), r, world, causal, scale)
           for r in range(world)]
    held = [(sh(k, r), sh(v, r)) + rbs[r].new_accumulators() for r in range(world)]
    for t in range(world):
        for r in range(world):
            rbs[r].consume(t, *held[r])
        held = [held[(r - 1) % world] for r in range(world)]  # shards and their accumulators move on
    grads = [rbs[r].finish(held[r][2], held[r][3]) for r in range(world)]  # each shard is home again
    return [torch.cat([g[i] for g in grads]) for i in range(3)]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("S", [128, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_attention_backward_emulated(fa, world, S, d, causal):
    from _gpu import GRAD_TOL, rel_l2
    inp = workloads.random_inputs(2, d, "bf16", seed=950 + world + S + d + int(causal), B=1, N=world * S,
                                  causal=causal)
    dev = torch.device("cuda")
    q, k, v, do = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.do.to(dev)
    o, lse = _ring_local(fa, q, k, v, world, causal, inp.scale)
    dq, dk, dv = _ring_local_bwd(q, k, v, o, lse, do, world, causal, inp.scale)
    ref = oracle.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        assert rel_l2(f64(g), r) <= GRAD_TOL, (name, rel_l2(f64(g), r))


def test_ring_attention_backward_matches_single_call(fa):
    """4 ranks × 1024 tokens, causal, d = 128: the ring's gradients against the oracle and against the
    single-call backward of the whole sequence."""
    from _gpu import GRAD_TOL, rel_l2
    world, S = 4, 1024
    inp = workloads.random_inputs(2, 128, "bf16", seed=4343, B=1, N=world * S, causal=True)
    dev = torch.device("cuda")
    q, k, v, do = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.do.to(dev)
    o, lse = _ring_local(fa, q, k, v, world, True, inp.scale)
    g_ring = _ring_local_bwd(q, k, v, o, lse, do, world, True, inp.scale)
    ref = oracle.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.scale, True)
    o1, l1 = fa.attention_forward(q, k, v, causal=True, scale=inp.scale)
    g_one = fa.attention_backward(q, k, v, o1, l1, do, causal=True, scale=inp.scale)
    for a, b, r in zip(g_ring, g_one, ref):
        assert rel_l2(f64(a), r) <= GRAD_TOL and rel_l2(f64(a), f64(b)) <= GRAD_TOL


# ----------------------------------------------------------------------------- load-balanced (zigzag) layout


def _ring_zigzag(q, k, v, do, world, causal, scale):
    """The zigzag ring, forward and (with do) backward, ranks side by side; results in sequence order."""
    from exact_io_aware_90_b200.ring import RingAttention, RingAttentionBackward, zigzag_shard, zigzag_unshard
    sh = lambda x, r: zigzag_shard(x, r, world)
    ras = [RingAttention(sh(q, r), r, world, causal, scale, layout="zigzag") for r in range(world)]
    held = [(sh(k, r), sh(v, r)) for r in range(world)]
    for t in range(world):
        for r in range(world):
            ras[r].consume(t, *held[r])
        held = [held[(r - 1) % world] for r in range(world)]
    outs = [ra.result() for ra in ras]
    o, lse = zigzag_unshard([x for x, _ in outs]), zigzag_unshard([x for _, x in outs])
    if do is None:
        return o, lse, None
    rbs = [RingAttentionBackward(sh(q, r), outs[r][0], outs[r][1], sh(do, r), r, world, causal, scale,
                                 layout="zigzag") for r in range(world)]
    held = [(sh(k, r), sh(v, r)) + rbs[r].new_accumulators() for r in range(world)]
    for t in range(world):
        for r in range(world):
            rbs[r].consume(t, *held[r])
        held = [held[(r - 1) % world] for r in range(world)]
    grads = [rbs[r].finish(held[r][2], held[r][3]) for r in range(world)]
    return o, lse, [zigzag_unshard([g[i] for g in grads]) for i in range(3)]


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("C", [64, 150])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_zigzag_ring_emulated(fa, world, C, d, causal):
    """The load-balanced ring (chunks r and 2W−1−r per rank, chunk-pair blocks) against the oracle's
    attention and gradients over the whole sequence."""
    from _gpu import GRAD_TOL, rel_l2
    L = 2 * world * C
    inp = workloads.random_inputs(2, d, "bf16", seed=970 + world + C + d + int(causal), B=1, N=L, causal=causal)
    dev = torch.device("cuda")
    q, k, v, do = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.do.to(dev)
    o, lse, grads = _ring_zigzag(q, k, v, do, world, causal, inp.scale)
    O_ref, L_ref = oracle.attention_forward(inp.q, inp.k, inp.v, inp.scale, causal)
    assert max_abs(f64(o), O_ref) <= O_TOL
    assert max_abs(f64(lse), L_ref) <= LSE_TOL
    ref = oracle.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), grads, ref):
        assert rel_l2(f64(g), r) <= GRAD_TOL, (name, rel_l2(f64(g), r))
