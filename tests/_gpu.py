"""Helpers for the GPU parity tests: run the CUDA path through the binding and
compare with the fp64 oracle on the same (already rounded) inputs.

Tolerances (bf16/fp16 inputs, fp32 accumulation):
  max |O - O_ref|     <= 1e-2
  max |LSE - LSE_ref| <= 1e-3
  relative L2 error of dQ, dK, dV <= 2e-2  (||x - x_ref||_2 / ||x_ref||_2)
"""

import numpy as np
import torch

import oracle

O_TOL = 1e-2
LSE_TOL = 1e-3
GRAD_TOL = 2e-2


def f64(t):
    return t.detach().float().cpu().double().numpy()


def max_abs(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


def rel_l2(a, b):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


def gpu_forward(fa, inp, out=None, lse=None):
    dev = torch.device("cuda")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    o, l = fa.attention_forward(q, k, v, causal=inp.causal, scale=inp.scale, cu_seqlens=cu,
                                max_seqlen=inp.N if cu is not None else None, batch=inp.B, out=out, lse=lse)
    st = fa.fa_check_device_status(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return o, l


def gpu_backward(fa, inp, o, lse):
    dev = torch.device("cuda")
    q, k, v, do = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev), inp.do.to(dev)
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    dq, dk, dv = fa.attention_backward(q, k, v, o, lse, do, causal=inp.causal, scale=inp.scale, cu_seqlens=cu,
                                       max_seqlen=inp.N if cu is not None else None, batch=inp.B)
    st = fa.fa_check_device_status(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return dq, dk, dv


def covered_rows(inp):
    """Token rows that belong to some sequence."""
    if inp.cu_seqlens is None:
        return np.arange(inp.T)
    cu = inp.cu_seqlens.numpy()
    return np.concatenate([np.arange(cu[b], cu[b + 1]) for b in range(len(cu) - 1)] + [np.zeros(0, int)])


def oracle_forward(inp):
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return oracle.attention_forward(inp.q, inp.k, inp.v, inp.scale, inp.causal, cu_seqlens=cu, B=inp.B,
                                    N=inp.N if cu is None else None)


def oracle_backward(inp):
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.numpy()
    return oracle.attention_backward(inp.q, inp.k, inp.v, inp.do, inp.scale, inp.causal, cu_seqlens=cu, B=inp.B,
                                     N=inp.N if cu is None else None)
