"""GPU parity of the e4m3 forward (fa_fwd_fp8) against the fp64 oracle, through the C ABI.

The inputs are e4m3 tensors with per-tensor descales (``workloads.random_inputs(..., "e4m3")``); the
oracle computes the plain definition on the real values (stored value × descale).  The kernel's only
rounding beyond fp32 is that of P to e4m3 before P·V (3 mantissa bits: relative error ≤ 2⁻⁴; values
below the smallest subnormal 2⁻⁹ of the row's reference maximum flush, absolute error ≤ 2⁻¹⁰, and
the softmax sum ℓ relative to that maximum is ≥ 1) and that of O to bf16.  So, per element,

    |O − O_ref|_ic ≤ 2⁻⁴·Σ_j P_ij |v_jc| + Σ_j min(P_ij, 2⁻¹⁰)·|v_jc| + 2⁻⁸·|O_ref,ic| + 1e-4,

and, the roundings being independent and centred, the RMS error over a tensor is at most about
σ = 2⁻⁴/√3 · sqrt(mean Σ_j P_ij² v_jc²) (checked with a factor 1.5).  For random values that noise is
a few percent of |O| per element, so a systematic error (a misapplied scale or descale) is caught by
the least-squares factor of O on O_ref, which must be 1 within five standard errors σ/(rms O_ref·√n).
LSE involves no e4m3 rounding: the plain 1e-3 bound.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from _gpu import LSE_TOL, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    m.fa_set_watchdog_ns(2_000_000_000)
    return m


def _real(inp):
    if "descale_blk" in inp.extra:  # one descale per (128-token block, head)
        ds, segs = inp.extra["descale_blk"], workloads.block_segments(_seq_bounds(inp))
        return tuple(workloads.real_values(t, ds[n], segs) for t, n in ((inp.q, "q"), (inp.k, "k"), (inp.v, "v")))
    if "descale_bh" in inp.extra:  # one descale per (sequence, head)
        ds, segs = inp.extra["descale_bh"], _seq_bounds(inp)
        return tuple(workloads.real_values(t, ds[n], segs) for t, n in ((inp.q, "q"), (inp.k, "k"), (inp.v, "v")))
    ds = inp.extra["descale"]
    return (workloads.real_values(inp.q, ds["q"]), workloads.real_values(inp.k, ds["k"]),
            workloads.real_values(inp.v, ds["v"]))


def _run(fa, inp, **over):
    dev = torch.device("cuda")
    per_block = "descale_blk" in inp.extra
    if per_block or "descale_bh" in inp.extra:
        ds = {n: torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)
              for n, a in inp.extra["descale_blk" if per_block else "descale_bh"].items()}
    else:
        ds = dict(inp.extra["descale"], **over)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    o, lse = fa.attention_forward_fp8(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), ds["q"], ds["k"], ds["v"],
                                      causal=inp.causal, scale=inp.scale, cu_seqlens=cu,
                                      max_seqlen=inp.N if cu is not None else None, batch=inp.B,
                                      per_block=per_block)
    assert fa.fa_check_device_status(torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    return o, lse


def _v_descale_per_token(inp):
    """[T, H] descale of v at every token (None when v has one descale per tensor or per sequence, where
    the plain bound below applies)."""
    if "descale_blk" not in inp.extra:
        return None
    out = np.ones((inp.T, inp.H))
    for (s0, L), ds in zip(workloads.block_segments(_seq_bounds(inp)), inp.extra["descale_blk"]["v"]):
        out[s0:s0 + L] = ds[None, :]
    return out


def _seq_bounds(inp):
    """(start, length) of every sequence."""
    if inp.cu_seqlens is None:
        return [(b * inp.N, inp.N) for b in range(inp.B)]
    cu = inp.cu_seqlens.tolist()
    return [(cu[b], cu[b + 1] - cu[b]) for b in range(len(cu) - 1)]


def _rounding_terms(q, k, v, lse_ref, scale, causal, seqs, rows=None, vd=None):
    """For the chosen tokens (all heads): A = Σ_j P|v|, Bt = Σ_j min(P, 2⁻¹⁰)|v|, Q2 = Σ_j P²v², with P
    from the oracle's LSE (P_ij = exp(scale·q_i·k_j − LSE_i) over the visible keys).

    With v descales that differ between key blocks (``vd`` [T, H], the descale of each key) the kernel
    rounds P_ij·vd_j / W_i, with W_i ≤ M_i = max_j P_ij·vd_j (its row maximum is that of the weighted
    values), so the flush term becomes Bt = Σ_j min(P_ij|v_j|, 2⁻¹⁰·M_i·|v_j| / vd_j)."""
    T, H, d = q.shape
    A, Bt, Q2 = (np.zeros((T, H, d)) for _ in range(3))
    want = np.ones(T, dtype=bool) if rows is None else np.isin(np.arange(T), rows)
    for s0, L in seqs:
        toks = [t for t in range(s0, s0 + L) if want[t]]
        if not toks:
            continue
        ti = np.array(toks)
        for h in range(H):
            S = scale * q[ti, h, :] @ k[s0:s0 + L, h, :].T                      # [rows, L]
            P = np.exp(S - lse_ref[ti, h][:, None])
            if causal:
                P = np.where(np.arange(L)[None, :] <= (ti - s0)[:, None], P, 0.0)
            va = np.abs(v[s0:s0 + L, h, :])
            A[ti, h] = P @ va
            if vd is None:
                Bt[ti, h] = np.minimum(P, 2.0 ** -10) @ va
            else:
                w = vd[s0:s0 + L, h]                                              # [L]
                M = np.max(P * w[None, :], axis=1, keepdims=True)                 # [rows, 1]
                Bt[ti, h] = np.sum(np.minimum(P[:, :, None] * va[None], 2.0 ** -10 * M[:, :, None]
                                              * (va / w[:, None])[None]), axis=1)
            Q2[ti, h] = (P * P) @ (va * va)
    return A, Bt, Q2


def _check(inp, o, lse, rows=None):
    q, k, v = _real(inp)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    if rows is None:
        O_ref, L_ref = oracle.attention_forward(q, k, v, inp.scale, inp.causal, cu_seqlens=cu, B=inp.B,
                                                N=inp.N if cu is None else None)
        sel = np.ones(inp.T, dtype=bool)
    else:
        O_r, L_r = oracle.attention_forward_rows(q, k, v, rows, inp.scale, inp.causal, cu_seqlens=cu, B=inp.B,
                                                 N=inp.N if cu is None else None)
        O_ref, L_ref = np.zeros(q.shape), np.zeros(q.shape[:2])
        O_ref[rows], L_ref[rows] = O_r, L_r
        sel = np.isin(np.arange(inp.T), rows)
    A, Bt, Q2 = _rounding_terms(q, k, v, L_ref, inp.scale, inp.causal, _seq_bounds(inp), rows,
                                vd=_v_descale_per_token(inp))
    got, gl = f64(o)[sel], f64(lse)[sel]
    err = np.abs(got - O_ref[sel])
    bound = 2.0 ** -4 * A[sel] + Bt[sel] + 2.0 ** -8 * np.abs(O_ref[sel]) + 1e-4
    worst = np.unravel_index(np.argmax(err - bound), err.shape) if err.size else None
    assert np.all(err <= bound), (err[worst], bound[worst])
    if err.size:
        ref = O_ref[sel]
        rms = math.sqrt(float(np.mean(err ** 2)))
        rms_pred = 2.0 ** -4 / math.sqrt(3.0) * math.sqrt(float(np.mean(Q2[sel])))
        rms_ref = math.sqrt(float(np.mean(ref ** 2)))
        rms_out = 2.0 ** -9 * rms_ref
        assert rms <= 1.5 * rms_pred + rms_out + 1e-5, (rms, rms_pred, rms_out)
        # no systematic error: the least-squares factor of the output on the reference is 1 within five
        # standard errors of the rounding noise (a misapplied scale or descale moves it by far more)
        if rms_ref > 0:
            alpha = float(np.sum(got * ref) / np.sum(ref * ref))
            assert abs(alpha - 1.0) <= 5.0 * rms_pred / (rms_ref * math.sqrt(ref.size)) + 2.0 ** -10, alpha
        assert float(np.max(np.abs(gl - L_ref[sel]))) <= LSE_TOL
    return err


@pytest.mark.parametrize("N", [1, 63, 129, 300, 700])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_forward(fa, N, causal):
    inp = workloads.random_inputs(2, 128, "e4m3", seed=500 + N + int(causal), B=2, N=N, causal=causal,
                                  backward=False)
    o, lse = _run(fa, inp)
    assert o.dtype == torch.bfloat16
    _check(inp, o, lse)


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_varlen(fa, causal):
    inp = workloads.random_inputs(3, 128, "e4m3", seed=77, seqlens=[5, 0, 257, 130, 1030], causal=causal,
                                  backward=False)
    o, lse = _run(fa, inp)
    _check(inp, o, lse)


def test_fp8_descales_fold_exactly(fa):
    """Powers of two moved between the q and k descales leave every score unchanged, and doubling v's
    descale doubles O: both exactly, since the kernel only multiplies by them."""
    inp = workloads.random_inputs(2, 128, "e4m3", seed=9, B=1, N=520, causal=True, backward=False)
    ds = inp.extra["descale"]
    o1, l1 = _run(fa, inp)
    o2, l2 = _run(fa, inp, q=ds["q"] * 4.0, k=ds["k"] / 4.0)
    o3, l3 = _run(fa, inp, v=ds["v"] * 2.0)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o3.float(), 2.0 * o1.float()) and torch.equal(l1, l3)


def test_fp8_full_size_sampled_rows(fa):
    """The measured workload (B=4, H=16, N=8192, d=128, causal), in the launch configuration the
    benchmark times, on 48 seeded rows (all heads) against the oracle's row-restricted forward."""
    inp = workloads.make_workload("causal_n8k_d128_fp8")
    o, lse = _run(fa, inp)
    rng = np.random.default_rng(5)
    rows = np.sort(np.concatenate([rng.choice(inp.T, 40, replace=False), [0, 127, 128, 8191, 8192, 16383, 24576,
                                                                             inp.T - 1]]))
    rows = np.unique(rows)
    _check(inp, o, lse, rows=rows)


@pytest.mark.parametrize("varlen", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_per_head_descales(fa, causal, varlen):
    """One descale per (sequence, head) (fa_fwd_fp8_per_head): heads and sequences drawn at magnitudes
    a factor 2 apart, each quantised with its own amax/448, so a kernel that used one descale for all
    would be far off; checked under the same e4m3 bounds against the oracle on the real values."""
    H, d = 3, 128
    seqlens = [200, 0, 513, 64] if varlen else [384, 384]
    B, N = len(seqlens), max(seqlens)
    cu = workloads.cu_from_lengths(seqlens) if varlen else None
    segs = [(int(sum(seqlens[:b])), L) for b, L in enumerate(seqlens)]
    T = sum(seqlens)
    g = torch.Generator().manual_seed(61 + int(causal) + 2 * int(varlen))
    mag = torch.ones(T, H, 1)
    for b, (s0, L) in enumerate(segs):
        mag[s0:s0 + L] = (2.0 ** torch.arange(H, dtype=torch.float32))[None, :, None] * (b + 1)
    q8, dq = workloads.quantize_e4m3_per_head(torch.randn(T, H, d, generator=g) * mag, segs)
    k8, dk = workloads.quantize_e4m3_per_head(torch.randn(T, H, d, generator=g) * mag, segs)
    v8, dv = workloads.quantize_e4m3_per_head(torch.randn(T, H, d, generator=g) * mag, segs)
    inp = workloads.AttnInputs(q8, k8, v8, None, cu, seqlens, B, H, N, d, 0.25 / math.sqrt(d), causal, "e4m3",
                               "per_head", {"descale_bh": {"q": dq, "k": dk, "v": dv}})
    o, lse = _run(fa, inp)
    _check(inp, o, lse)


def _per_block_inputs(seqlens, varlen, causal, seed, H=3, d=128):
    """e4m3 inputs with one descale per (128-token block, head): every block and head drawn at its own
    magnitude (factors of 2 and 3 apart along heads and blocks, so that one descale per sequence would
    be far off) and quantised with its own amax/448."""
    B, N = len(seqlens), max(seqlens)
    cu = workloads.cu_from_lengths(seqlens) if varlen else None
    segs = [(int(sum(seqlens[:b])), L) for b, L in enumerate(seqlens)]
    T = sum(seqlens)
    g = torch.Generator().manual_seed(seed)
    mags = []
    for name in ("q", "k", "v"):
        mag = torch.ones(T, H, 1)
        for n, (s0, L) in enumerate(workloads.block_segments(segs)):
            mag[s0:s0 + L] = (2.0 ** torch.arange(H, dtype=torch.float32))[None, :, None] * (1 + (n + len(name)) % 3)
        mags.append(mag)
    (q8, dq), (k8, dk), (v8, dv) = (workloads.quantize_e4m3_per_block(torch.randn(T, H, d, generator=g) * m, segs)
                                    for m in mags)
    return workloads.AttnInputs(q8, k8, v8, None, cu, seqlens, B, H, N, d, 0.25 / math.sqrt(d), causal, "e4m3",
                                "per_block", {"descale_blk": {"q": dq, "k": dk, "v": dv}})


@pytest.mark.parametrize("varlen", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_per_block_descales(fa, causal, varlen):
    """One descale per (128-token block, head) (fa_fwd_fp8_per_block): q's per query tile, k's per key
    tile, v's carried in P, against the oracle on the real values under the e4m3 bounds (the flush term
    with the weighted row maximum).  The lengths leave ragged last blocks, an empty sequence, and a
    sequence of one tile."""
    seqlens = [200, 0, 513, 64] if varlen else [384, 384]
    inp = _per_block_inputs(seqlens, varlen, causal, seed=71 + int(causal) + 2 * int(varlen))
    o, lse = _run(fa, inp)
    _check(inp, o, lse)


def test_fp8_per_block_equal_descales_match_per_tensor(fa):
    """Per-block descales that are all equal compute exactly what the per-tensor call computes (the
    same folded constant, log2 of the descale added to m and subtracted again through ℓ): compared
    against fa_fwd_fp8 within the e4m3 rounding of a different but equivalent exponent split."""
    inp = workloads.random_inputs(2, 128, "e4m3", seed=19, B=2, N=700, causal=True, backward=False)
    ds = inp.extra["descale"]
    nb = 2 * ((700 + 127) // 128)
    blk = {n: np.full((nb, 2), np.float32(ds[n]), dtype=np.float32) for n in ("q", "k", "v")}
    o1, l1 = _run(fa, inp)
    pb = workloads.AttnInputs(inp.q, inp.k, inp.v, None, None, inp.seqlens, inp.B, inp.H, inp.N, inp.d, inp.scale,
                              inp.causal, "e4m3", "per_block", {"descale_blk": blk})
    o2, l2 = _run(fa, pb)
    _check(pb, o2, l2)
    assert float((o1.float() - o2.float()).abs().max()) <= 2.0 ** -3 * float(o1.float().abs().max())
    assert float((l1 - l2).abs().max()) <= 1e-4


def test_fp8_per_block_too_few_blocks_is_reported(fa):
    """Varlen with descale arrays one block short: the host cannot count the blocks, so the kernel finds
    the last sequence's blocks past the arrays, skips that sequence and records FA_ERR_INVALID_ARG; the
    other sequences are computed as usual."""
    seqlens = [130, 300]
    inp = _per_block_inputs(seqlens, True, True, seed=5)
    dev = torch.device("cuda")
    ds = {n: torch.from_numpy(np.ascontiguousarray(a[:-1], dtype=np.float32)).to(dev)
          for n, a in inp.extra["descale_blk"].items()}
    o = torch.full((inp.T, inp.H, inp.d), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((inp.T, inp.H), 7.0, dtype=torch.float32, device=dev)
    fa.attention_forward_fp8(inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), ds["q"], ds["k"], ds["v"], causal=True,
                             scale=inp.scale, cu_seqlens=inp.cu_seqlens.to(dev), max_seqlen=inp.N, batch=inp.B,
                             out=o, lse=lse, per_block=True)
    stream = torch.cuda.current_stream().cuda_stream
    assert fa.fa_check_device_status(stream) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_check_device_status(stream) == fa.FA_OK  # reading the status clears it
    assert bool((o[130:].float() == 7.0).all()) and bool((lse[130:] == 7.0).all())  # skipped: untouched
    q, k, v = _real(inp)
    O_ref, L_ref = oracle.attention_forward(q[:130], k[:130], v[:130], inp.scale, True, B=1, N=130)
    assert float(np.max(np.abs(f64(lse[:130]) - L_ref))) <= LSE_TOL
    assert float(np.max(np.abs(f64(o[:130]) - O_ref))) <= 0.1 * float(np.max(np.abs(O_ref)))


def test_fp8_per_block_many_sequences(fa):
    """Per-block descales with 41 sequences: each softmax warp counts the blocks of the sequences before
    its unit's in chunks of 32 (one per lane), so a batch past 32 sequences takes the chunk loop more
    than once; lengths include 0, 1, 128 and 129."""
    g = torch.Generator().manual_seed(404)
    seqlens = [int(x) for x in torch.randint(0, 300, (37,), generator=g)] + [0, 1, 128, 129]
    inp = _per_block_inputs(seqlens, True, True, seed=405, H=2)
    o, lse = _run(fa, inp)
    _check(inp, o, lse)
