"""B200-native exact attention (forward and recomputing backward) for sm_100a.

This package is a thin Python binding over ``libfa_b200.so`` — the C ABI
declared in ``include/fa.h``.  Every step of the computation runs in the
library's CUDA kernels; Python only marshals arguments (device pointers, sizes,
the current CUDA stream) and, in the convenience wrappers, allocates output
tensors with PyTorch.  There is no fallback: if the library is missing or no
GPU is present the calls raise.

Raw ABI (same names and argument order as ``include/fa.h``; pointers are ints):
    fa_fwd, fa_bwd, fa_bwd_preprocess, fa_bwd_main, fa_bwd_postprocess,
    fa_bwd_workspace_bytes, fa_bwd_noalloc, fa_fwd_dropout, fa_bwd_dropout, fa_fwd_fp8, fa_fwd_fp8_per_head, fa_attn_merge, fa_accumulate,
    fa_decode,
    fa_decode_workspace_bytes, fa_check_device_status, fa_set_watchdog_ns, fa_watchdog_selftest, fa_status_string, fa_version
Torch wrappers:
    attention_forward(q, k, v, ...)          -> (o, lse)
    attention_backward(q, k, v, o, lse, do, ...) -> (dq, dk, dv)
    attention_decode(q, k, v, ...)           -> (o, lse)   one query per sequence over a K/V cache
    attention_forward_fp8(q8, k8, v8, descales, ...) -> (o bf16, lse)   e4m3 inputs
    attention_merge(acc_o, acc_lse, part_o, part_lse, ...)   merge a partial (O, LSE) into a running result
Ring (context-parallel) attention over a process group: ``exact_io_aware_90_b200.ring``.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

__all__ = [
    "FAError", "LIB_PATH", "lib", "FA_OK", "FA_ERR_INVALID_ARG", "FA_ERR_UNSUPPORTED", "FA_ERR_CUDA",
    "FA_ERR_TIMEOUT", "FA_BF16", "FA_FP16",
    "fa_fwd", "fa_bwd", "fa_bwd_preprocess", "fa_bwd_main", "fa_bwd_postprocess", "fa_bwd_workspace_bytes",
    "fa_bwd_noalloc", "FA_NOALLOC_SCRATCH_BYTES", "fa_fwd_dropout", "fa_bwd_dropout", "fa_fwd_fp8", "fa_fwd_fp8_per_head", "fa_attn_merge", "fa_accumulate", "fa_decode", "fa_decode_workspace_bytes", "fa_check_device_status", "fa_set_watchdog_ns", "fa_watchdog_selftest", "fa_status_string", "fa_version",
    "attention_forward", "attention_backward", "attention_decode", "attention_forward_fp8", "attention_merge", "dtype_code",
]

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT = 0, 1, 2, 3, 4
FA_BF16, FA_FP16 = 0, 1
FA_NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # include/fa.h

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {fa_status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python exact_io_aware_90_b200/build.py` "
            "(nvcc, sm_100a). There is no fallback implementation.")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, S, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "fa_fwd": (I, [P, P, P, P, P, I, I, I, I, F, I, P, I, I, P]),
        "fa_bwd_workspace_bytes": (S, [I, I, I]),
        "fa_bwd": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, I, I, P, S, P]),
        "fa_bwd_preprocess": (I, [P, P, I, I, I, I, P, I, I, P, S, P]),
        "fa_bwd_main": (I, [P, P, P, P, P, P, P, I, I, I, I, F, I, P, I, I, P, S, P]),
        "fa_bwd_postprocess": (I, [P, I, I, I, I, F, P, I, I, P, S, P]),
        "fa_bwd_noalloc": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, I, I, P]),
        "fa_fwd_dropout": (I, [P, P, P, P, P, I, I, I, I, F, I, P, I, I, F, U64, ctypes.c_uint32, P]),
        "fa_bwd_dropout": (I, [P, P, P, P, P, P, P, P, P, I, I, I, I, F, I, P, I, I, F, U64, ctypes.c_uint32, P, S,
                               P]),
        "fa_fwd_fp8": (I, [P, P, P, P, P, I, I, I, I, F, I, P, I, F, F, F, P]),
        "fa_fwd_fp8_per_head": (I, [P, P, P, P, P, I, I, I, I, F, I, P, I, P, P, P, P]),
        "fa_fwd_fp8_per_block": (I, [P, P, P, P, P, I, I, I, I, F, I, P, I, P, P, P, I, P]),
        "fa_attn_merge": (I, [P, P, P, P, P, I, I, I, I, I, P]),
        "fa_accumulate": (I, [P, P, P, ctypes.c_longlong, I, I, P]),
        "fa_decode_workspace_bytes": (S, [I, I, I, I]),
        "fa_decode": (I, [P, P, P, P, P, I, I, I, I, F, P, I, I, P, S, P]),
        "fa_check_device_status": (I, [P]),
        "fa_set_watchdog_ns": (None, [U64]),
        "fa_watchdog_selftest": (I, [U64, P]),
        "fa_status_string": (ctypes.c_char_p, [I]),
        "fa_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    return L


lib = _load()


# ----------------------------------------------------------------------------- raw ABI (ints for pointers)

def fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, stream) -> int:
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, stream)


def fa_bwd_workspace_bytes(total_tokens, H, d) -> int:
    return lib.fa_bwd_workspace_bytes(total_tokens, H, d)


def fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype,
           workspace, workspace_bytes, stream) -> int:
    return lib.fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype,
                      workspace, workspace_bytes, stream)


def fa_bwd_preprocess(o, dO, B, H, N, d, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes, stream) -> int:
    return lib.fa_bwd_preprocess(o, dO, B, H, N, d, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes,
                                 stream)


def fa_bwd_main(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, workspace,
                workspace_bytes, stream) -> int:
    return lib.fa_bwd_main(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype,
                           workspace, workspace_bytes, stream)


def fa_bwd_postprocess(dq, B, H, N, d, scale, cu_seqlens, total_tokens, dtype, workspace, workspace_bytes,
                       stream) -> int:
    return lib.fa_bwd_postprocess(dq, B, H, N, d, scale, cu_seqlens, total_tokens, dtype, workspace,
                                  workspace_bytes, stream)


def fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype,
                   stream) -> int:
    """fa_bwd with its workspace in the library's static device scratch, for callers that cannot
    allocate device memory; limited to problems needing at most FA_NOALLOC_SCRATCH_BYTES of
    scratch (see include/fa.h)."""
    return lib.fa_bwd_noalloc(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens,
                              dtype, stream)


def fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, dropout_p, seed,
                   offset, stream) -> int:
    return lib.fa_fwd_dropout(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype, dropout_p,
                              seed, offset, stream)


def fa_bwd_dropout(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens, dtype,
                   dropout_p, seed, offset, workspace, workspace_bytes, stream) -> int:
    return lib.fa_bwd_dropout(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, cu_seqlens, total_tokens,
                              dtype, dropout_p, seed, offset, workspace, workspace_bytes, stream)


def fa_fwd_fp8(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale, k_descale,
               v_descale, stream) -> int:
    return lib.fa_fwd_fp8(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale, k_descale,
                          v_descale, stream)


def fa_fwd_fp8_per_head(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale, k_descale,
                        v_descale, stream) -> int:
    return lib.fa_fwd_fp8_per_head(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale,
                                   k_descale, v_descale, stream)


def fa_fwd_fp8_per_block(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale, k_descale,
                         v_descale, num_blocks, stream) -> int:
    return lib.fa_fwd_fp8_per_block(q, k, v, o, lse, B, H, N, d, scale, causal, cu_seqlens, total_tokens, q_descale,
                                    k_descale, v_descale, num_blocks, stream)


def fa_attn_merge(acc_o, acc_lse, part_o, part_lse, out, T, H, d, dtype, first, stream) -> int:
    return lib.fa_attn_merge(acc_o, acc_lse, part_o, part_lse, out, T, H, d, dtype, first, stream)


def fa_accumulate(acc, part, out, n, dtype, first, stream) -> int:
    return lib.fa_accumulate(acc, part, out, n, dtype, first, stream)


def fa_decode_workspace_bytes(B, H, Nk, d) -> int:
    return lib.fa_decode_workspace_bytes(B, H, Nk, d)


def fa_decode(q, k, v, o, lse, B, H, Nk, d, scale, cu_seqlens_k, total_keys, dtype, workspace, workspace_bytes,
              stream) -> int:
    return lib.fa_decode(q, k, v, o, lse, B, H, Nk, d, scale, cu_seqlens_k, total_keys, dtype, workspace,
                         workspace_bytes, stream)


def fa_check_device_status(stream) -> int:
    return lib.fa_check_device_status(stream)


def fa_set_watchdog_ns(ns: int) -> None:
    lib.fa_set_watchdog_ns(int(ns))


def fa_watchdog_selftest(timeout_ns: int, stream) -> int:
    return lib.fa_watchdog_selftest(int(timeout_ns), stream)


def fa_status_string(status: int) -> str:
    return lib.fa_status_string(int(status)).decode()


def fa_version() -> str:
    return lib.fa_version().decode()


# ----------------------------------------------------------------------------- torch wrappers

def dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"unsupported dtype {t.dtype}: q/k/v must be bfloat16 or float16")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _shape(q, cu_seqlens, max_seqlen, batch):
    T, H, d = q.shape
    if cu_seqlens is None:
        B = 1 if batch is None else int(batch)
        if T % B:
            raise ValueError("token count must be a multiple of the batch size")
        N = T // B
    else:
        B = int(cu_seqlens.numel()) - 1
        if max_seqlen is None:
            raise ValueError("max_seqlen is required with cu_seqlens")
        N = int(max_seqlen)
    return B, H, N, d, T


def _check(t, name, q):
    if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype or t.shape != q.shape:
        raise ValueError(f"{name} must be a contiguous CUDA tensor like q")


def attention_forward(q, k, v, causal: bool = False, scale: Optional[float] = None, cu_seqlens=None,
                      max_seqlen: Optional[int] = None, batch: Optional[int] = None, out=None, lse=None,
                      stream=None, dropout_p: float = 0.0, seed: int = 0,
                      offset: int = 0) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """O and LSE for q, k, v of shape [T, H, d] (see ``include/fa.h``); ``dropout_p`` > 0 drops
    probabilities with the in-kernel mask of (seed, offset)."""
    import torch
    for t, n in ((k, "k"), (v, "v")):
        _check(t, n, q)
    _check(q, "q", q)
    B, H, N, d, T = _shape(q, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    if dropout_p:
        st = lib.fa_fwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, float(scale),
                                int(bool(causal)), _ptr(cu_seqlens), T, dtype_code(q), float(dropout_p), int(seed),
                                int(offset), stream)
    else:
        st = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, float(scale), int(bool(causal)),
                        _ptr(cu_seqlens), T, dtype_code(q), stream)
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return out, lse


def attention_backward(q, k, v, o, lse, do, causal: bool = False, scale: Optional[float] = None, cu_seqlens=None,
                       max_seqlen: Optional[int] = None, batch: Optional[int] = None, dq=None, dk=None, dv=None,
                       workspace=None, stream=None, dropout_p: float = 0.0, seed: int = 0, offset: int = 0):
    """dq, dk, dv for the forward that produced (o, lse) (with the same dropout_p, seed, offset)."""
    import torch
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _check(t, n, q)
    _check(q, "q", q)
    B, H, N, d, T = _shape(q, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = lib.fa_bwd_workspace_bytes(T, H, d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    if dropout_p:
        st = lib.fa_bwd_dropout(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv),
                                B, H, N, d, float(scale), int(bool(causal)), _ptr(cu_seqlens), T, dtype_code(q),
                                float(dropout_p), int(seed), int(offset), _ptr(workspace),
                                workspace.numel() * workspace.element_size(), stream)
    else:
        st = lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                        N, d, float(scale), int(bool(causal)), _ptr(cu_seqlens), T, dtype_code(q), _ptr(workspace),
                        workspace.numel() * workspace.element_size(), stream)
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def attention_forward_fp8(q, k, v, q_descale: float, k_descale: float, v_descale: float, causal: bool = False,
                          scale: Optional[float] = None, cu_seqlens=None, max_seqlen: Optional[int] = None,
                          batch: Optional[int] = None, out=None, lse=None, stream=None, per_block: bool = False):
    """O (bf16) and LSE for e4m3 q, k, v of shape [T, H, 128] whose real values are the stored ones times
    the descales: floats (one per tensor, fa_fwd_fp8), fp32 CUDA tensors [B, H] (one per sequence and
    head, fa_fwd_fp8_per_head) or, with ``per_block``, fp32 CUDA tensors [num_blocks, H] (one per
    128-token block of each sequence and head, fa_fwd_fp8_per_block); see ``include/fa.h``."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.float8_e4m3fn or t.shape != q.shape:
            raise ValueError(f"{n} must be a contiguous CUDA float8_e4m3fn tensor shaped like q")
    B, H, N, d, T = _shape(q, cu_seqlens, max_seqlen, batch)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, H, d), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((T, H), dtype=torch.float32, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    per_head = [hasattr(x, "data_ptr") for x in (q_descale, k_descale, v_descale)]
    if per_block:
        if not all(per_head):
            raise ValueError("per-block descales must be [num_blocks, H] tensors")
        nb = q_descale.numel() // H
        for x in (q_descale, k_descale, v_descale):
            if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous() or x.numel() != nb * H or nb < 1:
                raise ValueError("per-block descales must be contiguous CUDA float32 tensors of num_blocks·H values")
        st = lib.fa_fwd_fp8_per_block(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, float(scale),
                                      int(bool(causal)), _ptr(cu_seqlens), T, _ptr(q_descale), _ptr(k_descale),
                                      _ptr(v_descale), nb, stream)
    elif any(per_head):
        if not all(per_head):
            raise ValueError("the three descales must all be floats or all be [B, H] tensors")
        for x in (q_descale, k_descale, v_descale):
            if not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous() or x.numel() != B * H:
                raise ValueError("per-head descales must be contiguous CUDA float32 tensors of B·H values")
        st = lib.fa_fwd_fp8_per_head(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, float(scale),
                                     int(bool(causal)), _ptr(cu_seqlens), T, _ptr(q_descale), _ptr(k_descale),
                                     _ptr(v_descale), stream)
    else:
        st = lib.fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, N, d, float(scale),
                            int(bool(causal)), _ptr(cu_seqlens), T, float(q_descale), float(k_descale), float(v_descale),
                            stream)
    if st != FA_OK:
        raise FAError(st, "fa_fwd_fp8")
    return out, lse


def attention_merge(acc_o, acc_lse, part_o, part_lse, out=None, first: bool = False, stream=None):
    """Merge the normalised partial (part_o [T, H, d] bf16/fp16, part_lse [T, H] fp32) into the running
    result (acc_o fp32 [T, H, d], acc_lse fp32 [T, H]); with ``out`` the merged O goes there in
    part_o's dtype (see ``include/fa.h``, fa_attn_merge)."""
    import torch
    T, H, d = part_o.shape
    for t, n, dt in ((acc_o, "acc_o", torch.float32), (acc_lse, "acc_lse", torch.float32),
                     (part_lse, "part_lse", torch.float32)):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != dt:
            raise ValueError(f"{n} must be a contiguous CUDA {dt} tensor")
    if acc_o.shape != part_o.shape or acc_lse.shape != (T, H) or part_lse.shape != (T, H):
        raise ValueError("acc_o must be [T, H, d] and the LSE arrays [T, H], as part_o")
    if out is not None and (out.shape != part_o.shape or out.dtype != part_o.dtype or not out.is_contiguous()):
        raise ValueError("out must be a contiguous tensor like part_o")
    if stream is None:
        stream = torch.cuda.current_stream(part_o.device).cuda_stream
    st = lib.fa_attn_merge(_ptr(acc_o), _ptr(acc_lse), _ptr(part_o), _ptr(part_lse), _ptr(out), T, H, d,
                           dtype_code(part_o), int(bool(first)), stream)
    if st != FA_OK:
        raise FAError(st, "fa_attn_merge")


def attention_decode(q, k, v, scale: Optional[float] = None, cu_seqlens_k=None, max_seqlen_k: Optional[int] = None,
                     out=None, lse=None, workspace=None, stream=None):
    """O [B, H, d] and LSE [B, H] of one query per sequence (q: [B, H, d]) over its keys in
    k, v: [Tk, H, d] (see ``include/fa.h``).  Without ``cu_seqlens_k`` the Tk = B·Nk keys
    form B sequences of Nk keys."""
    import torch
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
            raise ValueError(f"{n} must be a contiguous CUDA tensor with q's dtype")
    B, H, d = q.shape
    Tk = k.shape[0]
    if k.shape != (Tk, H, d) or v.shape != k.shape:
        raise ValueError("k and v must be [Tk, H, d] with q's H and d")
    if cu_seqlens_k is None:
        if Tk % B:
            raise ValueError("key count must be a multiple of the batch size")
        Nk = Tk // B
    else:
        if int(cu_seqlens_k.numel()) != B + 1:
            raise ValueError("cu_seqlens_k needs B + 1 entries")
        if max_seqlen_k is None:
            raise ValueError("max_seqlen_k is required with cu_seqlens_k")
        Nk = int(max_seqlen_k)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = lib.fa_decode_workspace_bytes(B, H, Nk, d)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if stream is None:
        stream = torch.cuda.current_stream(q.device).cuda_stream
    st = lib.fa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nk, d, float(scale),
                       _ptr(cu_seqlens_k), Tk, dtype_code(q), _ptr(workspace),
                       workspace.numel() * workspace.element_size(), stream)
    if st != FA_OK:
        raise FAError(st, "fa_decode")
    return out, lse
