"""GPU parity of dropout on P (forward and backward) against the fp64 oracle, through the C ABI.

The keep mask is drawn inside the kernels from Philox4x32-10; the oracle draws it from its own
implementation of the same generator (pinned by the generator's known-answer vectors), so the
masks must agree bit for bit: one test reads the mask out exactly (V = identity makes O = dropped P).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from _gpu import GRAD_TOL, LSE_TOL, O_TOL, covered_rows, f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    m.fa_set_watchdog_ns(2_000_000_000)
    return m


def _p32(p):
    return float(np.float32(p))  # the value the C ABI receives


def _o_tol(p):
    # the kept terms are amplified by 1/(1 − p), and so is the output's rounding to bf16/fp16 (row 0 of a causal
    # head is 2·v_0 at p = 0.5): the plain bound holds for (1 − p)·O, the output before the amplification
    return O_TOL / (1.0 - _p32(p))


def _dev(inp):
    dev = torch.device("cuda")
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    kw = dict(causal=inp.causal, scale=inp.scale, cu_seqlens=cu, max_seqlen=inp.N if cu is not None else None,
              batch=inp.B)
    return inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), kw


def _oracle_kw(inp):
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return dict(cu_seqlens=cu, B=inp.B, N=inp.N if cu is None else None)


@pytest.mark.parametrize("N", [1, 63, 129, 300])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("p", [0.1, 0.5])
def test_dropout_forward_backward(fa, N, d, causal, p):
    inp = workloads.random_inputs(2, d, "bf16", seed=N + d + int(causal), B=2, N=N, causal=causal)
    q, k, v, kw = _dev(inp)
    seed, off = 0x9E3779B97F4A7C15, 3
    o, lse = fa.attention_forward(q, k, v, dropout_p=p, seed=seed, offset=off, **kw)
    s = torch.cuda.current_stream().cuda_stream
    assert fa.fa_check_device_status(s) == fa.FA_OK
    O_ref, L_ref = oracle.attention_forward_dropout(inp.q, inp.k, inp.v, inp.scale, causal, _p32(p), seed, off,
                                                    **_oracle_kw(inp))
    assert max_abs(f64(o), O_ref) <= _o_tol(p), max_abs(f64(o), O_ref)
    assert max_abs(f64(lse), L_ref) <= LSE_TOL
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, inp.do.to(q.device), dropout_p=p, seed=seed, offset=off,
                                       **kw)
    assert fa.fa_check_device_status(s) == fa.FA_OK
    g_ref = oracle.attention_backward_dropout(inp.q, inp.k, inp.v, inp.do, inp.scale, causal, _p32(p), seed, off,
                                              **_oracle_kw(inp))
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        if name in ("dq", "dk") and N == 1:
            # one key: dS = P∘(dP − D) is exactly 0, so dQ = dK = 0.  The kernel's D = Σ_c dO_c·O_c uses the
            # output rounded to bf16 (relative error ≤ 2⁻⁹, |O_c| ≤ |v_c|/(1 − p)), so |dS| ≤ Σ_c |dO_c v_c|·2⁻⁹/(1 − p),
            # |dQ| ≤ scale·|dS|·max|k| and |dK| ≤ scale·|dS|·max|q|; the bound doubles that for fp32 accumulation
            dov = (np.abs(f64(inp.do)) * np.abs(f64(inp.v))).sum(axis=-1).max()  # N = 1: row t's key is token t
            other = inp.k if name == "dq" else inp.q
            bound = inp.scale * dov / (1 - p) * 2.0 ** -8 * np.abs(f64(other)).max()
            assert np.abs(f64(g)).max() <= bound, (np.abs(f64(g)).max(), bound)
            continue
        e = rel_l2(f64(g), r)
        assert e <= GRAD_TOL, (name, e)


def test_dropout_varlen(fa):
    inp = workloads.random_inputs(3, 128, "fp16", seed=12, seqlens=[5, 0, 257, 130], causal=True)
    q, k, v, kw = _dev(inp)
    o, lse = fa.attention_forward(q, k, v, dropout_p=0.25, seed=77, offset=1, **kw)
    O_ref, L_ref = oracle.attention_forward_dropout(inp.q, inp.k, inp.v, inp.scale, True, 0.25, 77, 1,
                                                    **_oracle_kw(inp))
    rows = covered_rows(inp)
    assert max_abs(f64(o)[rows], O_ref[rows]) <= _o_tol(0.25) and max_abs(f64(lse)[rows], L_ref[rows]) <= LSE_TOL
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, inp.do.to(q.device), dropout_p=0.25, seed=77, offset=1, **kw)
    g_ref = oracle.attention_backward_dropout(inp.q, inp.k, inp.v, inp.do, inp.scale, True, 0.25, 77, 1,
                                              **_oracle_kw(inp))
    for g, r in zip((dq, dk, dv), g_ref):
        assert rel_l2(f64(g)[rows], r[rows]) <= GRAD_TOL


def _mask_case(causal):
    """B = 2 sequences × H = 2 heads of N = 256 tokens, d = 128: two query tiles and two key tiles per
    (sequence, head), and four values of the head index b·H + h in the Philox counter."""
    B, H, N, d = 2, 2, 256, 128
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B * N, H, d, generator=g).to(torch.bfloat16)
    k = torch.randn(B * N, H, d, generator=g).to(torch.bfloat16)
    visible = np.tril(np.ones((N, N), dtype=bool)) if causal else np.ones((N, N), dtype=bool)
    return B, H, N, d, q, k, visible, 1.0 / math.sqrt(d), (0.375, 1234567, 9)


def _window_eye(B, H, N, d, w0):
    """[B·N, H, d] with token w0 + c of every sequence carrying e_c (c < d), all other tokens 0."""
    x = torch.zeros(B * N, H, d, dtype=torch.bfloat16)
    for b in range(B):
        x[b * N + w0 + torch.arange(d), :, torch.arange(d)] = 1.0
    return x


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_mask_is_exact(fa, causal):
    """V carries e_c on key w0 + c: O[i, c] is the dropped, rescaled P[i, w0 + c], so every kept and
    every dropped element of the forward kernel's mask over that key window is visible and must
    equal the oracle's mask exactly (and hidden keys must give exact zeros)."""
    B, H, N, d, q, k, visible, scale, (p, seed, off) = _mask_case(causal)
    dev = torch.device("cuda")
    t = oracle.dropout_threshold(_p32(p))
    for w0 in (0, N - d):
        v = _window_eye(B, H, N, d, w0)
        o, _ = fa.attention_forward(q.to(dev), k.to(dev), v.to(dev), causal=causal, scale=scale, batch=B,
                                    dropout_p=p, seed=seed, offset=off)
        got = f64(o)
        for b in range(B):
            for h in range(H):
                keep = oracle.dropout_keep_mask(N, b * H + h, seed, off, t)[:, w0:w0 + d]
                vis = visible[:, w0:w0 + d]
                gbh = got[b * N:(b + 1) * N, h, :]
                assert np.array_equal(gbh[vis] != 0.0, keep[vis]), (w0, b, h)
                assert np.all(gbh[~vis] == 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_mask_is_exact(fa, causal):
    """dO carries e_c on query w0 + c: dV[j, c] = (dropped, rescaled P)[w0 + c, j], so the backward
    kernel's own regeneration of the mask is visible element by element over that query window."""
    B, H, N, d, q, k, visible, scale, (p, seed, off) = _mask_case(causal)
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(4)
    v = torch.randn(B * N, H, d, generator=g).to(torch.bfloat16)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o, lse = fa.attention_forward(qd, kd, vd, causal=causal, scale=scale, batch=B, dropout_p=p, seed=seed,
                                  offset=off)
    t = oracle.dropout_threshold(_p32(p))
    for w0 in (0, N - d):
        do = _window_eye(B, H, N, d, w0).to(dev)
        _, _, dv = fa.attention_backward(qd, kd, vd, o, lse, do, causal=causal, scale=scale, batch=B, dropout_p=p,
                                         seed=seed, offset=off)
        got = f64(dv)
        for b in range(B):
            for h in range(H):
                keep = oracle.dropout_keep_mask(N, b * H + h, seed, off, t)[w0:w0 + d, :].T  # [key j, query c]
                vis = visible[w0:w0 + d, :].T
                gbh = got[b * N:(b + 1) * N, h, :]
                assert np.array_equal(gbh[vis] != 0.0, keep[vis]), (w0, b, h)
                assert np.all(gbh[~vis] == 0.0)


def test_dropout_zero_is_plain(fa):
    inp = workloads.random_inputs(2, 128, "bf16", seed=4, B=1, N=300, causal=True)
    q, k, v, kw = _dev(inp)
    o1, l1 = fa.attention_forward(q, k, v, **kw)
    o1, l1 = o1.clone(), l1.clone()
    s = torch.cuda.current_stream().cuda_stream
    o2, l2 = torch.empty_like(o1), torch.empty_like(l1)
    st = fa.fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), 1, 2, 300, 128,
                           inp.scale, 1, None, 300, fa.FA_BF16, 0.0, 5, 0, s)
    assert st == fa.FA_OK and fa.fa_check_device_status(s) == fa.FA_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
