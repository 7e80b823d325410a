"""GPU parity of the backward kernels against the fp64 oracle (through the C ABI).

dQ, dK, dV must be within a relative L2 error of 2e-2 of the oracle's
gradients on the same rounded inputs (the GPU forward's O and LSE feed the
GPU backward, as in training).  Full-size workloads are checked on sampled
(sequence, head) pairs, which the oracle computes completely: a head's dK and
dV depend on that head alone.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads
from _gpu import GRAD_TOL, covered_rows, f64, gpu_backward, gpu_forward, oracle_backward, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    m.fa_set_watchdog_ns(2_000_000_000)
    return m


def _check_bwd(fa, inp, tol=GRAD_TOL):
    o, lse = gpu_forward(fa, inp)
    dq, dk, dv = gpu_backward(fa, inp, o, lse)
    rdq, rdk, rdv = oracle_backward(inp)
    rows = covered_rows(inp)
    errs = {}
    for name, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        a = f64(g)[rows]
        assert np.all(np.isfinite(a)), name
        errs[name] = rel_l2(a, r[rows])
    assert max(errs.values()) <= tol, errs
    return errs


@pytest.mark.parametrize("N", [1, 3, 64, 127, 128, 129, 200, 257, 511])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes_bf16(fa, N, d, causal):
    inp = workloads.random_inputs(2, d, "bf16", seed=31 * N + d + int(causal), B=2, N=N, causal=causal)
    _check_bwd(fa, inp)


@pytest.mark.parametrize("N", [64, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_small_shapes_fp16(fa, N, d, causal):
    inp = workloads.random_inputs(2, d, "fp16", seed=17 * N + d + int(causal), B=1, N=N, causal=causal)
    _check_bwd(fa, inp)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_varlen_ragged(fa, d, causal):
    lens = [1, 127, 128, 129, 0, 300, 1030, 5]
    inp = workloads.random_inputs(2, d, "bf16", seed=41 + d, seqlens=lens, causal=causal)
    _check_bwd(fa, inp)


def test_gradient_sum_invariants(fa):
    """Σ_j dK_j ≈ 0 and Σ_j dV_j ≈ Σ_i dO_i per head (exact for the true gradients)."""
    inp = workloads.random_inputs(4, 128, "bf16", seed=77, B=1, N=640, causal=True)
    o, lse = gpu_forward(fa, inp)
    dq, dk, dv = gpu_backward(fa, inp, o, lse)
    dk_sum = f64(dk).sum(axis=0)
    dv_sum = f64(dv).sum(axis=0)
    do_sum = f64(inp.do).sum(axis=0)
    scale_dk = np.abs(f64(dk)).sum(axis=0)
    assert np.all(np.abs(dk_sum) <= 2e-2 * scale_dk + 1e-3)
    assert np.max(np.abs(dv_sum - do_sum)) <= 2e-2 * np.max(np.abs(do_sum)) + 0.05


def _sampled_heads(inp, n, seed):
    rng = np.random.default_rng(seed)
    pairs = [(b, h) for b in range(inp.B) for h in range(inp.H) if inp.seqlens[b] > 0]
    idx = rng.choice(len(pairs), size=min(n, len(pairs)), replace=False)
    return [pairs[i] for i in sorted(idx)]


@pytest.mark.parametrize("name,nheads", [("mha_n4k_d64", 3), ("causal_n8k_d128", 2), ("varlen_causal_d128", 3)])
def test_workload_backward_sampled_heads(fa, name, nheads):
    inp = workloads.make_workload(name, backward=True)
    o, lse = gpu_forward(fa, inp)
    dq, dk, dv = gpu_backward(fa, inp, o, lse)
    if inp.cu_seqlens is None:
        starts = [b * inp.N for b in range(inp.B)]
    else:
        starts = inp.cu_seqlens.tolist()[:-1]
    for b, h in _sampled_heads(inp, nheads, seed=len(name)):
        s, L = starts[b], inp.seqlens[b]
        sl = slice(s, s + L)
        sub = workloads.AttnInputs(inp.q[sl, h:h + 1], inp.k[sl, h:h + 1], inp.v[sl, h:h + 1],
                                   inp.do[sl, h:h + 1], None, [L], 1, 1, L, inp.d, inp.scale, inp.causal, inp.dtype)
        rdq, rdk, rdv = oracle_backward(sub)
        for nm, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            e = rel_l2(f64(g[sl, h:h + 1]), r)
            assert e <= GRAD_TOL, (name, b, h, nm, e)
