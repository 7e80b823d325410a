"""The e4m3 parity checks of tests/test_gpu_fp8.py, run on a CPU model of the kernel's arithmetic (no GPU).

The model takes the same steps as the e4m3 forward with per-block descales: per key tile j the softmax
constant c_j = scale·log2(e)·q_descale·k_descale_j, the exponent c_j·s + log2 v_descale_j − m with m the
row maximum of c_j·s + log2 v_descale_j, P rounded to e4m3 by torch's conversion, ℓ = Σ 2^(…)/v_descale_j,
O = Σ P_e4m3·v_stored / ℓ rounded to bf16, LSE = (m + log2 ℓ)·ln 2.  The checks must accept this model
(the derived bound admits a correct kernel) and reject it with any of three plausible mistakes — k's
descale 1 % off, v's descales left out, ℓ not divided by v's descale — (the bound is not so loose that a
wrong kernel passes).
"""

import math

import numpy as np
import pytest
import torch

import workloads
from test_gpu_fp8 import _check, _per_block_inputs, _seq_bounds


def _model(inp, mistake=None):
    ds = inp.extra["descale_blk"]
    blocks = workloads.block_segments(_seq_bounds(inp))
    T, H, d = inp.q.shape
    qs, ks, vs = (t.to(torch.float64).numpy() for t in (inp.q.float(), inp.k.float(), inp.v.float()))
    blk_of = np.zeros(T, dtype=np.int64)
    for n, (s0, L) in enumerate(blocks):
        blk_of[s0:s0 + L] = n
    o = np.zeros((T, H, d))
    lse = np.full((T, H), -np.inf)
    c0 = inp.scale * math.log2(math.e)
    for s0, L in _seq_bounds(inp):
        if L == 0:
            continue
        tok = np.arange(s0, s0 + L)
        for h in range(H):
            qd = ds["q"][blk_of[tok], h].astype(np.float64)
            kd = ds["k"][blk_of[tok], h].astype(np.float64)
            vd = ds["v"][blk_of[tok], h].astype(np.float64)
            if mistake == "k_descale_off":
                kd = kd * 1.01
            S = qs[tok, h] @ ks[tok, h].T                                   # stored-value scores
            x = c0 * qd[:, None] * kd[None, :] * S
            lv = np.log2(vd)
            if mistake != "v_descale_ignored":
                x = x + lv[None, :]
            if inp.causal:
                x = np.where(np.arange(L)[None, :] <= np.arange(L)[:, None], x, -np.inf)
            m = x.max(axis=1, keepdims=True)
            e = np.exp2(x - m)
            pe = torch.from_numpy(e).to(torch.float8_e4m3fn).to(torch.float64).numpy()
            den = vd if mistake not in ("no_v_in_sum", "v_descale_ignored") else np.ones_like(vd)
            ell = (e / den[None, :]).sum(axis=1)
            out = pe @ vs[tok, h] / ell[:, None]
            o[tok, h] = out
            lse[tok, h] = (m[:, 0] + np.log2(ell)) * math.log(2.0)
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).to(torch.float32)


@pytest.mark.parametrize("varlen", [False, True])
@pytest.mark.parametrize("causal", [False, True])
def test_per_block_checks_accept_the_model(causal, varlen):
    inp = _per_block_inputs([200, 0, 513, 64] if varlen else [384, 384], varlen, causal, seed=71 + int(causal))
    o, lse = _model(inp)
    _check(inp, o, lse)


@pytest.mark.parametrize("mistake", ["k_descale_off", "v_descale_ignored", "no_v_in_sum"])
def test_per_block_checks_reject_a_wrong_model(mistake):
    inp = _per_block_inputs([384, 384], False, True, seed=72)
    o, lse = _model(inp, mistake)
    with pytest.raises(AssertionError):
        _check(inp, o, lse)
