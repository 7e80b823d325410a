"""Seeded synthetic inputs for the attention workloads.

Shared by the tests, ``bench.py`` and ``__graft_entry__``.  This module holds
none of the attention arithmetic: it only draws i.i.d. N(0, 1) numbers from a
seeded CPU generator, rounds them to the storage dtype, draws sequence lengths
and builds the ``cu_seqlens`` prefix array.  Both the CUDA path and the fp64
oracle consume exactly the tensors made here (the oracle widens the rounded
values to float64).

Layout: q, k, v, dO are [T, H, d] row-major; ``cu_seqlens`` is int32 [B+1]
or None (then T = B·N).  The workloads are the five measured shapes:

==================  =========================================================
name                shape
==================  =========================================================
tiny_d64            B=1, H=1, N=256, d=64, bf16, non-causal, forward only
mha_n4k_d64         B=8, H=16, N=4096, d=64, fp16, non-causal, fwd+bwd
causal_n8k_d128     B=4, H=16, N=8192, d=128, bf16, causal, fwd+bwd
varlen_causal_d128  32 sequences, lengths uniform in [128, 4096], H=32,
                    d=128, bf16, causal, fwd+bwd
long_n128k_d128     B=1, H=8, N=131072, d=128, bf16, causal, forward only
causal_n8k_d128_fp8 B=4, H=16, N=8192, d=128, e4m3 (per-tensor descales),
                    causal, forward only
==================  =========================================================

e4m3 inputs: each tensor is drawn in fp32, divided by its descale
amax/448 (so its largest magnitude maps to e4m3's largest finite value) and
rounded to float8_e4m3fn; ``extra["descale"]`` holds the three descales and
the real value of an element is its e4m3 value times its tensor's descale.

Decode inputs (one query token per sequence over a K/V cache): q is
[B, H, d], k and v are [Tk, H, d] with ``cu_seqlens_k`` (or Tk = B·Nk):

==================  =========================================================
decode_b16_kv8k     B=16, H=16, Nk=8192 keys each, d=128, bf16
decode_varlen       64 sequences, key counts uniform in [512, 16384], H=16,
                    d=128, bf16
==================  =========================================================
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch

WORKLOADS = {
    "tiny_d64": dict(B=1, H=1, N=256, d=64, dtype="bf16", causal=False, backward=False, seed=1001),
    "mha_n4k_d64": dict(B=8, H=16, N=4096, d=64, dtype="fp16", causal=False, backward=True, seed=1002),
    "causal_n8k_d128": dict(B=4, H=16, N=8192, d=128, dtype="bf16", causal=True, backward=True, seed=1003),
    "varlen_causal_d128": dict(nseq=32, lmin=128, lmax=4096, H=32, d=128, dtype="bf16", causal=True,
                               backward=True, seed=1004),
    "long_n128k_d128": dict(B=1, H=8, N=131072, d=128, dtype="bf16", causal=True, backward=False, seed=1005),
    "causal_n8k_d128_fp8": dict(B=4, H=16, N=8192, d=128, dtype="e4m3", causal=True, backward=False, seed=1008),
}

TORCH_DTYPES = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclass
class AttnInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    do: Optional[torch.Tensor]
    cu_seqlens: Optional[torch.Tensor]  # int32 [B+1] or None
    seqlens: List[int]
    B: int
    H: int
    N: int            # maximum sequence length
    d: int
    scale: float
    causal: bool
    dtype: str
    name: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return int(self.q.shape[0])

    def to(self, device) -> "AttnInputs":
        mv = lambda t: None if t is None else t.to(device)
        return AttnInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.do), mv(self.cu_seqlens),
                          list(self.seqlens), self.B, self.H, self.N, self.d, self.scale, self.causal,
                          self.dtype, self.name, dict(self.extra))


E4M3_MAX = 448.0  # largest finite float8_e4m3fn value


def _randn(g: torch.Generator, shape, dtype: str) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(TORCH_DTYPES[dtype])


def _randn_e4m3(g: torch.Generator, shape):
    """(e4m3 tensor, descale) with real values = e4m3 value × descale, descale = amax / 448."""
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    descale = float(np.float32(float(x.abs().max()) / E4M3_MAX))  # the fp32 value the C ABI receives
    if not descale > 0.0:
        descale = 1.0  # an all-zero tensor keeps descale 1 (the C ABI wants it finite and > 0)
    return (x / descale).to(torch.float8_e4m3fn), descale


def real_values(t: torch.Tensor, descale=1.0, segments=None) -> np.ndarray:
    """The values a stored tensor stands for, as float64 (e4m3 or 16-bit storage times its descale):
    ``descale`` a float, or an [S, H] array with ``segments`` the (start, length) of each of the S
    token ranges it covers (sequences, or the 128-token blocks of ``block_segments``)."""
    x = t.detach().cpu().to(torch.float64).numpy()
    if segments is None:
        return x * float(descale)
    ds = np.asarray(descale, dtype=np.float64)
    out = x.copy()
    for b, (s0, L) in enumerate(segments):
        out[s0:s0 + L] *= ds[b][None, :, None]
    return out


def quantize_e4m3_per_head(x: torch.Tensor, segments):
    """fp32 [T, H, d] → (e4m3 tensor, fp32 descales [B, H]): each (sequence, head) divided by its own
    amax/448 (rounded to fp32) and rounded to e4m3."""
    T, H, _ = x.shape
    ds = np.ones((len(segments), H), dtype=np.float32)
    y = torch.zeros_like(x)  # tokens outside every segment stay 0
    for b, (s0, L) in enumerate(segments):
        if L == 0:
            continue
        amax = x[s0:s0 + L].abs().amax(dim=(0, 2))                      # [H]
        d = (amax / E4M3_MAX).numpy().astype(np.float32)
        ds[b] = np.where(d > 0, d, np.float32(1.0))  # an all-zero head keeps descale 1 (finite and > 0)
        y[s0:s0 + L] = x[s0:s0 + L] / torch.from_numpy(ds[b])[None, :, None]
    return y.to(torch.float8_e4m3fn), ds


def block_segments(segments, block: int = 128):
    """(start, length) of every 128-token block, sequence after sequence: block i of a sequence is its
    tokens [128i, 128i + 128), the last one ragged (the numbering of per-block e4m3 descales)."""
    return [(s0 + i, min(block, L - i)) for s0, L in segments for i in range(0, L, block)]


def quantize_e4m3_per_block(x: torch.Tensor, segments):
    """fp32 [T, H, d] → (e4m3 tensor, fp32 descales [num_blocks, H]): each (128-token block, head) of
    every sequence divided by its own amax/448 and rounded to e4m3; the real values follow from
    ``real_values(t, descales, block_segments(segments))``."""
    return quantize_e4m3_per_head(x, block_segments(segments))


def varlen_lengths(nseq: int, lmin: int, lmax: int, seed: int) -> List[int]:
    """Sequence lengths drawn uniformly from the integers [lmin, lmax]."""
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lmin, lmax + 1, size=nseq)]


def cu_from_lengths(lengths: List[int]) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def random_inputs(H: int, d: int, dtype: str, seed: int, *, B: int = 1, N: int = 0,
                  seqlens: Optional[List[int]] = None, causal: bool = False,
                  backward: bool = True, scale: Optional[float] = None, name: str = "") -> AttnInputs:
    """i.i.d. N(0,1) q, k, v (and dO) for a dense [B·N] or a packed (``seqlens``) batch."""
    if seqlens is not None:
        cu = cu_from_lengths(seqlens)
        T, B, N = int(cu[-1]), len(seqlens), max(seqlens) if seqlens else 0
    else:
        cu, T, seqlens = None, B * N, [N] * B
    g = torch.Generator().manual_seed(seed)
    extra = {}
    if dtype == "e4m3":
        if backward:
            raise ValueError("e4m3 inputs are forward only")
        (q, dq_), (k, dk_), (v, dv_) = (_randn_e4m3(g, (T, H, d)) for _ in range(3))
        extra["descale"] = {"q": dq_, "k": dk_, "v": dv_}
        if scale is None:
            scale = 1.0 / math.sqrt(d)
        return AttnInputs(q, k, v, None, cu, list(seqlens), B, H, N, d, float(scale), bool(causal), dtype, name,
                          extra)
    q = _randn(g, (T, H, d), dtype)
    k = _randn(g, (T, H, d), dtype)
    v = _randn(g, (T, H, d), dtype)
    do = None
    if backward:
        g2 = torch.Generator().manual_seed(seed + 1)
        do = _randn(g2, (T, H, d), dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return AttnInputs(q, k, v, do, cu, list(seqlens), B, H, N, d, float(scale), bool(causal), dtype, name)


def make_workload(name: str, backward: Optional[bool] = None) -> AttnInputs:
    """Inputs of one of the named workloads (on the CPU)."""
    w = dict(WORKLOADS[name])
    bwd = w["backward"] if backward is None else backward
    if "nseq" in w:
        lens = varlen_lengths(w["nseq"], w["lmin"], w["lmax"], w["seed"])
        return random_inputs(w["H"], w["d"], w["dtype"], w["seed"], seqlens=lens, causal=w["causal"],
                             backward=bwd, name=name)
    return random_inputs(w["H"], w["d"], w["dtype"], w["seed"], B=w["B"], N=w["N"], causal=w["causal"],
                         backward=bwd, name=name)


def hand_example_inputs(dtype: str = "fp16", d: int = 64) -> AttnInputs:
    """The narration's worked example as an attention call (B=1, H=1, N=4).

    Every query row is (1/scale)·e₀, so scale·q·k_j equals the first feature of
    k_j; key j carries ln c_j in that feature with c = [1, 2, 4, 3], and value
    j carries [10, 20, 30, 40][j] in its first feature.  All other features are
    zero.  The exact non-causal answer in feature 0 is 29 for every row.
    """
    scale = 1.0 / math.sqrt(d)
    c = [1.0, 2.0, 4.0, 3.0]
    vals = [10.0, 20.0, 30.0, 40.0]
    q = torch.zeros(4, 1, d, dtype=torch.float64)
    k = torch.zeros(4, 1, d, dtype=torch.float64)
    v = torch.zeros(4, 1, d, dtype=torch.float64)
    q[:, 0, 0] = 1.0 / scale
    for j in range(4):
        k[j, 0, 0] = math.log(c[j])
        v[j, 0, 0] = vals[j]
    tdt = TORCH_DTYPES[dtype]
    return AttnInputs(q.to(tdt), k.to(tdt), v.to(tdt), None, None, [4], 1, 1, 4, d, scale, False, dtype,
                      "hand_example")


DECODE_WORKLOADS = {
    "decode_b16_kv8k": dict(B=16, H=16, Nk=8192, d=128, dtype="bf16", seed=1006),
    "decode_varlen": dict(nseq=64, lmin=512, lmax=16384, H=16, d=128, dtype="bf16", seed=1007),
}


@dataclass
class DecodeInputs:
    q: torch.Tensor                      # [B, H, d]
    k: torch.Tensor                      # [Tk, H, d]
    v: torch.Tensor
    cu_seqlens_k: Optional[torch.Tensor]  # int32 [B+1] or None
    seqlens: List[int]                   # key count per sequence
    B: int
    H: int
    Nk: int                              # maximum key count
    d: int
    scale: float
    dtype: str
    name: str = ""

    @property
    def Tk(self) -> int:
        return int(self.k.shape[0])

    def to(self, device) -> "DecodeInputs":
        mv = lambda t: None if t is None else t.to(device)
        return DecodeInputs(mv(self.q), mv(self.k), mv(self.v), mv(self.cu_seqlens_k), list(self.seqlens), self.B,
                            self.H, self.Nk, self.d, self.scale, self.dtype, self.name)


def decode_inputs(H: int, d: int, dtype: str, seed: int, *, B: int = 1, Nk: int = 0,
                  seqlens: Optional[List[int]] = None, scale: Optional[float] = None, name: str = "") -> DecodeInputs:
    """i.i.d. N(0,1) q (one row per sequence), k and v for a dense or packed (``seqlens``) cache."""
    if seqlens is not None:
        cu = cu_from_lengths(seqlens)
        B, Tk, Nk = len(seqlens), int(cu[-1]), max(seqlens) if seqlens else 0
    else:
        cu, Tk, seqlens = None, B * Nk, [Nk] * B
    g = torch.Generator().manual_seed(seed)
    q = _randn(g, (B, H, d), dtype)
    k = _randn(g, (Tk, H, d), dtype)
    v = _randn(g, (Tk, H, d), dtype)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    return DecodeInputs(q, k, v, cu, list(seqlens), B, H, max(Nk, 1), d, float(scale), dtype, name)


def make_decode_workload(name: str) -> DecodeInputs:
    w = DECODE_WORKLOADS[name]
    if "nseq" in w:
        lens = varlen_lengths(w["nseq"], w["lmin"], w["lmax"], w["seed"])
        return decode_inputs(w["H"], w["d"], w["dtype"], w["seed"], seqlens=lens, name=name)
    return decode_inputs(w["H"], w["d"], w["dtype"], w["seed"], B=w["B"], Nk=w["Nk"], name=name)
