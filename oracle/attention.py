"""Plain fp64 CPU attention: the oracle that the CUDA path is checked against.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use it.  It shares no code with the CUDA library and imports
nothing from the ``exact_io_aware_90_b200`` package.

Everything here is deliberately slow and literal.  The method it checks
reaches the exact attention result, only reordered (FlashAttention 详解（零基础入门）,
§5.2 WARNING box: the rescaling is exact; FlashAttention 与算子融合, "online
softmax" paragraph: mathematically equivalent to the one-shot softmax;
FlashAttention 短片讲解稿, segment "适用范围与关键结论": same definition, not
bit-identical).  So the oracle is that definition written out in float64,
materialising the score matrix S and the probability matrix P for every
(sequence, head):

* scores   S = Q Kᵀ · scale                  (详解 §2.3, S = QKᵀ/√d)
* mask     S_ij = −∞ for key j > query i      (Flash Attention 优化, nanoGPT
                                               manual fallback: lower-triangular
                                               mask filled with −inf)
* softmax  P_ij = exp(S_ij − m_i) / Σ_k exp(S_ik − m_i), m_i = max_k S_ik
                                               (详解 §2.4, the safe form)
* output   O = P V                            (详解 §2.5)
* row log-sum-exp LSE_i = m_i + ln Σ_k exp(S_ik − m_i): the "few row
  statistics" the forward keeps for the backward (短片讲解稿, segment
  "第三招 · 反向重计算").

The backward is not printed on the pages; they only say that it recomputes P
from the inputs, the output and the row statistics (短片讲解稿 "第三招";
the foundit article: "反向传播也会重新计算部分中间值").  The oracle takes the
plainest reading, the chain rule applied to the four steps above:
dV = Pᵀ dO, dP = dO Vᵀ, D_i = Σ_j P_ij dP_ij, dS = P ∘ (dP − D), dQ = scale·dS K,
dK = scale·dSᵀ Q.

``online_blockwise_forward`` follows the tiled algorithm of 详解 §6.2 in the
pages' own order and notation (Q blocks outside, K/V blocks inside, running
m and ℓ, the normalised O update of §5.4).  It exists to pin the one-shot
definition against the pages' worked examples; the GPU is never compared
with it.

Tensor layout everywhere: [T, H, d] row-major (token, head, feature), T the
total token count; ``cu_seqlens`` (int, length B+1, starting at 0,
non-decreasing) packs B sequences of different lengths one after another
(FlashAttention 与算子融合, 工程实践 "变长序列 … varlen 接口（packing）").
Without ``cu_seqlens`` the T = B·N tokens form B sequences of N tokens.
"""

from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "sequence_segments",
    "attention_forward",
    "attention_backward",
    "attention_forward_rows",
    "attention_fwd_bwd_rows",
    "online_blockwise_forward",
    "online_softmax_stats",
    "merge_softmax_stats",
    "attention_flops",
    "decode_forward",
    "split_kv_decode",
    "merge_attention_partials",
    "zigzag_chunks",
    "ring_blocks",
    "ring_attention_forward",
    "ring_attention_backward",
    "philox4x32_10",
    "dropout_threshold",
    "dropout_keep_mask",
    "attention_forward_dropout",
    "attention_backward_dropout",
]


def _f64(x) -> np.ndarray:
    """Widen any array-like (numpy, or a CPU torch tensor) to float64 numpy."""
    if hasattr(x, "detach"):  # a torch tensor: widen through float32 (exact for 16-bit inputs)
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


def sequence_segments(T: int, B: int, N: int, cu_seqlens=None) -> List[Tuple[int, int]]:
    """(start token, length) of every sequence in the packed [T, H, d] layout."""
    if cu_seqlens is None:
        if T != B * N:
            raise ValueError(f"dense layout needs T == B*N, got T={T}, B={B}, N={N}")
        return [(b * N, N) for b in range(B)]
    cu = [int(c) for c in np.asarray(cu_seqlens).reshape(-1)]
    if len(cu) != B + 1 or cu[0] != 0:
        raise ValueError("cu_seqlens must have B+1 entries starting at 0")
    segs = []
    for b in range(B):
        if cu[b + 1] < cu[b]:
            raise ValueError("cu_seqlens must be non-decreasing")
        segs.append((cu[b], cu[b + 1] - cu[b]))
    if cu[B] > T:
        raise ValueError("cu_seqlens[B] exceeds the token count")
    return segs


def _scores(Q: np.ndarray, K: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """S = Q Kᵀ · scale with the causal mask applied (key j visible iff j <= i)."""
    S = (Q @ K.T) * scale
    if causal:
        L = S.shape[0]
        S[np.triu_indices(L, k=1)] = -np.inf
    return S


def _softmax_rows(S: np.ndarray):
    """Safe softmax along rows: returns P, the row max m and the row sum ℓ of exp(S - m)."""
    m = S.max(axis=1)
    E = np.exp(S - m[:, None])
    ell = E.sum(axis=1)
    P = E / ell[:, None]
    return P, m, ell


def attention_forward(q, k, v, scale: float, causal: bool = False, cu_seqlens=None,
                      B: Optional[int] = None, N: Optional[int] = None):
    """Exact attention forward in fp64.

    q, k, v: [T, H, d].  Returns (O [T, H, d] float64, LSE [T, H] float64).
    LSE is the natural-log log-sum-exp of the scaled, masked scores of each row.
    Tokens not covered by any sequence keep O = 0 and LSE = -inf.
    """
    Q, K, V = _f64(q), _f64(k), _f64(v)
    T, H, d = Q.shape
    if B is None:
        B = 1 if cu_seqlens is None else len(np.asarray(cu_seqlens)) - 1
    if N is None:
        N = T // B if cu_seqlens is None else 0
    O = np.zeros((T, H, d), dtype=np.float64)
    LSE = np.full((T, H), -np.inf, dtype=np.float64)
    for start, L in sequence_segments(T, B, N, cu_seqlens):
        if L == 0:
            continue
        sl = slice(start, start + L)
        for h in range(H):
            S = _scores(Q[sl, h], K[sl, h], scale, causal)
            P, m, ell = _softmax_rows(S)
            O[sl, h] = P @ V[sl, h]
            LSE[sl, h] = m + np.log(ell)
    return O, LSE


def attention_backward(q, k, v, do, scale: float, causal: bool = False, cu_seqlens=None,
                       B: Optional[int] = None, N: Optional[int] = None):
    """Gradients of L = <O, dO> with respect to q, k, v, in fp64.

    P is recomputed from the inputs (the plain definition, no tiling).
    Returns (dQ, dK, dV), each [T, H, d] float64.
    """
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(do)
    T, H, d = Q.shape
    if B is None:
        B = 1 if cu_seqlens is None else len(np.asarray(cu_seqlens)) - 1
    if N is None:
        N = T // B if cu_seqlens is None else 0
    dQ = np.zeros_like(Q)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    for start, L in sequence_segments(T, B, N, cu_seqlens):
        if L == 0:
            continue
        sl = slice(start, start + L)
        for h in range(H):
            S = _scores(Q[sl, h], K[sl, h], scale, causal)
            P, _, _ = _softmax_rows(S)
            g = dO[sl, h]
            dV[sl, h] = P.T @ g
            dP = g @ V[sl, h].T
            D = (P * dP).sum(axis=1)
            dS = P * (dP - D[:, None])  # masked entries have P = 0, so dS = 0 there
            dQ[sl, h] = scale * (dS @ K[sl, h])
            dK[sl, h] = scale * (dS.T @ Q[sl, h])
    return dQ, dK, dV


def attention_forward_rows(q, k, v, rows: Sequence[int], scale: float, causal: bool = False,
                           cu_seqlens=None, B: Optional[int] = None, N: Optional[int] = None):
    """O and LSE for a chosen set of query tokens only (all heads), in fp64.

    Each requested row is computed from its own sequence's keys, so the full
    [L, L] score matrix is never formed: this is how long sequences are
    checked on sampled rows.  Per (sequence, head) the sampled rows form a
    small [rows, L] score block with the same steps as ``attention_forward``.
    Returns (O [len(rows), H, d], LSE [len(rows), H]).
    """
    T, H, d = q.shape
    if B is None:
        B = 1 if cu_seqlens is None else len(np.asarray(cu_seqlens)) - 1
    if N is None:
        N = T // B if cu_seqlens is None else 0
    segs = sequence_segments(T, B, N, cu_seqlens)
    starts = np.array([s for s, _ in segs])
    rows = [int(r) for r in rows]
    O = np.zeros((len(rows), H, d), dtype=np.float64)
    LSE = np.full((len(rows), H), -np.inf, dtype=np.float64)
    by_seq = {}
    for n, t in enumerate(rows):
        b = int(np.searchsorted(starts, t, side="right")) - 1
        start, L = segs[b]
        if start <= t < start + L:
            by_seq.setdefault(b, []).append((n, t - start))
    for b, items in by_seq.items():
        start, L = segs[b]
        idx = np.array([n for n, _ in items])
        pos = np.array([i for _, i in items])
        hi = start + (int(pos.max()) + 1 if causal else L)  # keys any sampled row can see
        for h in range(H):
            Qr = _f64(q[start + pos, h] if not hasattr(q, "detach") else q[(start + pos).tolist(), h])
            Kh = _f64(k[start:hi, h])
            Vh = _f64(v[start:hi, h])
            S = (Qr @ Kh.T) * scale
            if causal:
                S[np.arange(Kh.shape[0])[None, :] > pos[:, None]] = -np.inf
            P, m, ell = _softmax_rows(S)
            O[idx, h] = P @ Vh
            LSE[idx, h] = m + np.log(ell)
    return O, LSE


def attention_fwd_bwd_rows(q, k, v, do, row_lo: int, row_hi: int, scale: float, causal: bool,
                           head: int = 0):
    """Forward and backward restricted to query rows [row_lo, row_hi) of one dense sequence.

    q, k, v, do: [L, H, d] for one sequence.  Returns (O, LSE, dQ) for the
    chosen rows and the partial (dK, dV) that those rows contribute to every
    key, all float64.  Used as a bounded CPU workload sample; it is the same
    arithmetic as ``attention_forward`` / ``attention_backward`` restricted to
    a block of rows.
    """
    Q = _f64(q[row_lo:row_hi, head])
    K = _f64(k[:, head])
    V = _f64(v[:, head])
    g = _f64(do[row_lo:row_hi, head])
    S = (Q @ K.T) * scale
    if causal:
        i = np.arange(row_lo, row_hi)[:, None]
        j = np.arange(K.shape[0])[None, :]
        S[j > i] = -np.inf
    P, m, ell = _softmax_rows(S)
    O = P @ V
    LSE = m + np.log(ell)
    dV = P.T @ g
    dP = g @ V.T
    D = (P * dP).sum(axis=1)
    dS = P * (dP - D[:, None])
    dQ = scale * (dS @ K)
    dK = scale * (dS.T @ Q)
    return O, LSE, dQ, dK, dV


def online_blockwise_forward(q, k, v, scale: float, causal: bool = False, bq: int = 64,
                             bk: int = 64, trace: Optional[list] = None):
    """The tiled forward of FlashAttention 详解 §6.2, taken step by step (one sequence).

    q: [N, H, d] or [N, d] (one head); k, v: the same with their own row count
    (equal to N when causal).  Block sizes need not divide the row counts;
    the last block is shorter (the pages use N // B blocks and are silent on
    remainders).  Q blocks are the outer loop, K/V blocks the inner loop; the
    running max m, the running sum ℓ and the output block are updated with the
    normalised rule of §5.4 / the §6.2 update line:
        m_new = max(m, rowmax(S_ij));  P_ij = exp(S_ij − m_new)
        ℓ_new = ℓ·exp(m − m_new) + rowsum(P_ij)
        O = O·(ℓ/ℓ_new)·exp(m − m_new) + P_ij V_j / ℓ_new
    A row that has seen only masked keys so far has m = −∞ and ℓ = 0; for it
    the correction factor is taken as 0 and O stays 0 (the pages are silent on
    this case; it needs a block whose keys are all hidden from the row).

    If ``trace`` is a list, (i, j, m_new, ℓ_new, numerator = O·ℓ_new) is
    appended after every inner step, so the pages' running numerator and
    denominator can be checked.  Returns (O, LSE) with the input's head shape.
    """
    Q, K, V = _f64(q), _f64(k), _f64(v)
    squeeze = Q.ndim == 2
    if squeeze:
        Q, K, V = Q[:, None, :], K[:, None, :], V[:, None, :]
    N, H, d = Q.shape
    Nk = K.shape[0]
    if causal and Nk != N:
        raise ValueError("the causal mask needs as many keys as queries")
    O = np.zeros((N, H, d))
    LSE = np.zeros((N, H))
    for h in range(H):
        for i0 in range(0, N, bq):
            i1 = min(i0 + bq, N)
            Qi = Q[i0:i1, h]
            Oi = np.zeros((i1 - i0, d))
            mi = np.full(i1 - i0, -np.inf)
            li = np.zeros(i1 - i0)
            for j0 in range(0, Nk, bk):
                j1 = min(j0 + bk, Nk)
                Kj, Vj = K[j0:j1, h], V[j0:j1, h]
                Sij = (Qi @ Kj.T) * scale
                if causal:
                    qi = np.arange(i0, i1)[:, None]
                    kj = np.arange(j0, j1)[None, :]
                    Sij = np.where(kj > qi, -np.inf, Sij)
                mij = Sij.max(axis=1)
                m_new = np.maximum(mi, mij)
                live = np.isfinite(m_new)
                shift = np.where(live, m_new, 0.0)
                Pij = np.where(live[:, None], np.exp(Sij - shift[:, None]), 0.0)
                corr = np.where(np.isfinite(mi), np.exp(mi - shift), 0.0)
                l_new = li * corr + Pij.sum(axis=1)
                safe_l = np.where(l_new > 0, l_new, 1.0)
                Oi = np.where(
                    (l_new > 0)[:, None],
                    Oi * (li / safe_l * corr)[:, None] + (Pij @ Vj) / safe_l[:, None],
                    0.0,
                )
                mi, li = m_new, l_new
                if trace is not None:
                    trace.append((i0 // bq, j0 // bk, mi.copy(), li.copy(), Oi * li[:, None]))
            O[i0:i1, h] = Oi
            LSE[i0:i1, h] = mi + np.log(li)
    if squeeze:
        return O[:, 0, :], LSE[:, 0]
    return O, LSE


def online_softmax_stats(x: Iterable[float], blocks: Sequence[int]):
    """Running (m, ℓ) of one row of scores fed in blocks of the given sizes.

    This is the two-statistic recurrence of 详解 §5.2:
        m⁽ᵗ⁾ = max(m⁽ᵗ⁻¹⁾, max_j x_j⁽ᵗ⁾)
        ℓ⁽ᵗ⁾ = ℓ⁽ᵗ⁻¹⁾·exp(m⁽ᵗ⁻¹⁾ − m⁽ᵗ⁾) + Σ_j exp(x_j⁽ᵗ⁾ − m⁽ᵗ⁾)
    Returns the list of (m, ℓ) after each block.
    """
    x = [float(t) for t in x]
    if sum(blocks) != len(x):
        raise ValueError("block sizes must add up to the row length")
    m, ell, out, pos = -math.inf, 0.0, [], 0
    for b in blocks:
        blk = x[pos:pos + b]
        pos += b
        m_new = max([m] + blk)
        ell = (ell * math.exp(m - m_new) if ell > 0 else 0.0) + sum(math.exp(t - m_new) for t in blk)
        m = m_new
        out.append((m, ell))
    return out


def merge_softmax_stats(m_a: float, l_a: float, m_b: float, l_b: float):
    """Merge two partial (max, sum) pairs: the form given by FlashAttention 与算子融合
    (online softmax paragraph): m = max(m_a, m_b), ℓ = ℓ_a·e^{m_a−m} + ℓ_b·e^{m_b−m}."""
    m = max(m_a, m_b)
    ell = 0.0
    if l_a > 0:
        ell += l_a * math.exp(m_a - m)
    if l_b > 0:
        ell += l_b * math.exp(m_b - m)
    return m, ell


def attention_flops(seqlens: Sequence[int], H: int, d: int, causal: bool, backward: bool = False) -> float:
    """Attention FLOPs by the convention of FlashAttention 与算子融合 (4·B·h·s²·d for
    the forward), summed over sequences, halved when causal; the backward counts
    2.5× the forward."""
    f = sum(4.0 * H * float(L) * float(L) * d for L in seqlens)
    if causal:
        f *= 0.5
    return f * 2.5 if backward else f


# ----------------------------------------------------------------------------- decode (one query per sequence)


def _key_segments(Tk: int, B: int, Nk: Optional[int], cu_seqlens_k) -> List[Tuple[int, int]]:
    if cu_seqlens_k is not None:
        cu = [int(c) for c in np.asarray(cu_seqlens_k).reshape(-1)]
        return [(cu[b], cu[b + 1]) for b in range(len(cu) - 1)]
    if Nk is None or B * Nk != Tk:
        raise ValueError("dense key layout needs B·Nk == Tk")
    return [(b * Nk, (b + 1) * Nk) for b in range(B)]


def decode_forward(q, k, v, scale: float, cu_seqlens_k=None, B: Optional[int] = None, Nk: Optional[int] = None):
    """Attention of one new query token per sequence over all keys of that sequence
    (token-by-token decoding, the workload FlashAttention 短片讲解稿 "适用范围与关键结论"
    sets apart): the same definition as ``attention_forward`` with a single query row
    and no mask, since every cached key precedes or is the current token.

    q: [B, H, d]; k, v: [Tk, H, d] with sequence b's keys at rows
    [cu_seqlens_k[b], cu_seqlens_k[b+1]) (or b·Nk … without cu_seqlens_k).
    Returns O [B, H, d] and LSE [B, H] (natural log) in float64; a sequence with
    no key gets O = 0 and LSE = −∞.
    """
    Q, K, V = _f64(q), _f64(k), _f64(v)
    Bq, H, d = Q.shape
    segs = _key_segments(K.shape[0], Bq if B is None else B, Nk, cu_seqlens_k)
    if len(segs) != Bq:
        raise ValueError("one query per sequence")
    O = np.zeros((Bq, H, d))
    LSE = np.full((Bq, H), -np.inf)
    for b, (lo, hi) in enumerate(segs):
        if hi <= lo:
            continue
        for h in range(H):
            s = (K[lo:hi, h] @ Q[b, h]) * scale          # [L] scores
            m = s.max()
            e = np.exp(s - m)
            O[b, h] = (e @ V[lo:hi, h]) / e.sum()
            LSE[b, h] = m + math.log(e.sum())
    return O, LSE


def split_kv_decode(q, k, v, scale: float, chunk: int, cu_seqlens_k=None, B: Optional[int] = None,
                    Nk: Optional[int] = None, return_partials: bool = False):
    """Decode by splitting each sequence's keys into chunks of ``chunk`` keys, each
    reduced on its own to a partial (m_c, ℓ_c, Õ_c = Σ_j e^{s_j − m_c} v_j), then
    merged in the form FlashAttention 与算子融合 gives for combining blocks
    ("FlashAttention 的两个关键", online softmax):
        m = max_c m_c,  ℓ = Σ_c ℓ_c·e^{m_c − m},  O = Σ_c Õ_c·e^{m_c − m} / ℓ
    (the output partial sums scaled the same way as ℓ).  Chunks are merged one at
    a time with ``merge_softmax_stats`` for (m, ℓ).  Mathematically equal to
    ``decode_forward``; it exists to pin the merge the GPU path performs.
    """
    Q, K, V = _f64(q), _f64(k), _f64(v)
    Bq, H, d = Q.shape
    segs = _key_segments(K.shape[0], Bq if B is None else B, Nk, cu_seqlens_k)
    O = np.zeros((Bq, H, d))
    LSE = np.full((Bq, H), -np.inf)
    partials = []
    for b, (lo, hi) in enumerate(segs):
        for h in range(H):
            m, ell, acc = -math.inf, 0.0, np.zeros(d)
            parts = []
            for c0 in range(lo, hi, chunk):
                c1 = min(hi, c0 + chunk)
                s = (K[c0:c1, h] @ Q[b, h]) * scale
                m_c = float(s.max())
                e = np.exp(s - m_c)
                l_c, O_c = float(e.sum()), e @ V[c0:c1, h]
                parts.append((m_c, l_c, O_c))
                m_new, ell = merge_softmax_stats(m, ell, m_c, l_c)
                acc = (acc * math.exp(m - m_new) if m > -math.inf else 0.0) + O_c * math.exp(m_c - m_new)
                m = m_new
            partials.append(parts)
            if ell > 0:
                O[b, h] = acc / ell
                LSE[b, h] = m + math.log(ell)
    if return_partials:
        return O, LSE, partials
    return O, LSE


# ----------------------------------------------------------------------------- partial results: merge, ring schedule


def merge_attention_partials(parts):
    """Combine attention results of the same queries over disjoint sets of keys.

    ``parts``: a list of (O_b, LSE_b) with O_b [..., d] normalised over its own keys and LSE_b [...]
    their natural-log sum of exponentials (−∞ where a part saw no key).  This is the block-merge rule
    of FlashAttention 与算子融合 ("FlashAttention 的两个关键", online softmax) for partials kept in
    normalised form: a normalised part is the pair (m, ℓ) = (LSE_b, 1) with Õ_b = O_b, so
        m = max_b LSE_b,  ℓ = Σ_b e^{LSE_b − m},  LSE = m + ln ℓ,  O = Σ_b e^{LSE_b − LSE} O_b.
    Parts are merged one at a time, as the ring schedule produces them.  Returns (O, LSE) in float64.
    """
    O = np.array(_f64(parts[0][0]), dtype=np.float64)
    L = np.array(_f64(parts[0][1]), dtype=np.float64)
    for Ob, Lb in parts[1:]:
        Ob, Lb = _f64(Ob), _f64(Lb)
        m = np.maximum(L, Lb)
        m_safe = np.where(np.isneginf(m), 0.0, m)          # both parts empty: keep LSE = −∞, O = 0
        ea, eb = np.exp(L - m_safe), np.exp(Lb - m_safe)    # e^{−∞} = 0 drops an empty part
        ell = ea + eb
        L_new = np.where(ell > 0, m_safe + np.log(np.where(ell > 0, ell, 1.0)), -np.inf)
        wa = np.where(ell > 0, ea / np.where(ell > 0, ell, 1.0), 0.0)
        wb = np.where(ell > 0, eb / np.where(ell > 0, ell, 1.0), 0.0)
        O = wa[..., None] * O + wb[..., None] * Ob
        L = L_new
    return O, L


def zigzag_chunks(rank: int, world: int):
    """Global chunk indices held by `rank` in the load-balanced ring layout: the sequence is cut into
    2·world equal chunks and rank r holds chunks r and 2·world − 1 − r (one from each end), so that under
    the causal mask every rank attends to as many keys as every other.  The pages name ring attention for
    very long sequences (FlashAttention 与算子融合, 工程实践 "与 CP 配合") but no shard order; this is the
    reading taken for a balanced one."""
    return (rank, 2 * world - 1 - rank)


def ring_blocks(rank: int, step: int, world: int, causal: bool, layout: str = "contiguous"):
    """The blocks rank `rank` computes at ring step `step`: a list of (query part, key part, causal
    diagonal?) over the parts of its own shard and of the shard it holds, that of rank
    s = (rank − step) mod world.  "contiguous": one part per shard (rank r holds positions [r·S, (r+1)·S));
    the block is the diagonal when s = r, skipped when s > r under the causal mask.  "zigzag": two parts
    per shard (``zigzag_chunks``); chunk pair (qc, kc) is the diagonal when qc = kc, skipped when
    kc > qc under the causal mask."""
    s_ = (rank - step) % world
    if layout == "contiguous":
        if causal and s_ > rank:
            return []
        return [(0, 0, causal and s_ == rank)]
    if layout != "zigzag":
        raise ValueError("layout must be 'contiguous' or 'zigzag'")
    out = []
    for qi, qc in enumerate(zigzag_chunks(rank, world)):
        for ki, kc in enumerate(zigzag_chunks(s_, world)):
            if causal and kc > qc:
                continue
            out.append((qi, ki, causal and kc == qc))
    return out


def _ring_parts(L: int, world: int, layout: str):
    """Row ranges of each rank's parts in the global sequence: parts[r] = [(start, stop), ...]."""
    if layout == "contiguous":
        if world < 1 or L % world:
            raise ValueError("the sequence must split into `world` equal shards")
        S = L // world
        return [[(r * S, (r + 1) * S)] for r in range(world)]
    if world < 1 or L % (2 * world):
        raise ValueError("the zigzag layout splits the sequence into 2·world equal chunks")
    C = L // (2 * world)
    return [[(c * C, (c + 1) * C) for c in zigzag_chunks(r, world)] for r in range(world)]


def ring_attention_forward(q, k, v, scale: float, causal: bool, world: int, layout: str = "contiguous"):
    """Attention of one dense sequence [L, H, d] computed as ring (context-parallel) attention over
    ``world`` ranks (FlashAttention 与算子融合, 工程实践: the ring of attention for very long
    sequences, with FlashAttention as the compute core): rank r holds positions [r·S, (r+1)·S),
    S = L / world, of q, k and v; at step t it holds the key/value shard of rank s = (r − t) mod
    world, attends its queries to it — the causal diagonal block when s = r, every key when s < r,
    nothing when s > r under the causal mask — and merges the block's (O, LSE) into its running
    result with ``merge_attention_partials``.  With ``layout="zigzag"`` each rank holds two chunks
    (``zigzag_chunks``) and computes the blocks ``ring_blocks`` lists, one running result per chunk.
    Returns (O [L, H, d], LSE [L, H]) in float64 in the sequence's own order, equal to
    ``attention_forward`` of the whole sequence."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    L, H, d = Q.shape
    parts_of = _ring_parts(L, world, layout)
    O = np.zeros((L, H, d))
    LSE = np.full((L, H), -np.inf)
    for r in range(world):
        partials = [[] for _ in parts_of[r]]
        for t in range(world):
            s_ = (r - t) % world
            for qi, ki, diag in ring_blocks(r, t, world, causal, layout):
                rows, cols = slice(*parts_of[r][qi]), slice(*parts_of[s_][ki])
                partials[qi].append(attention_forward(Q[rows], K[cols], V[cols], scale, diag))
        for qi, (a, b) in enumerate(parts_of[r]):
            O[a:b], LSE[a:b] = merge_attention_partials(partials[qi])
    return O, LSE


def ring_attention_backward(q, k, v, do, scale: float, causal: bool, world: int, layout: str = "contiguous"):
    """Gradients of ``ring_attention_forward`` computed on the same ring.  The probabilities of a block
    (query shard r, key shard s) are recomputed from the global row statistic, P_rs = exp(scale·Q_r K_sᵀ
    − LSE_r), as the tiled backward recomputes them from the saved LSE (FlashAttention 短片讲解稿,
    "第三招 · 反向重计算"), with D_r = Σ_c dO_rc·O_rc of the global output; then, per block,
        dS = P_rs ∘ (dO_r V_sᵀ − D_r),  dQ_r += scale·dS K_s,  dK_s += scale·dSᵀ Q_r,  dV_s += P_rsᵀ dO_r,
    where dQ_r accumulates on rank r and dK_s, dV_s travel with the key/value shard s around the ring
    and are home after one more step.  ``layout`` as in ``ring_attention_forward`` (blocks are then
    pairs of chunks).  Returns (dQ, dK, dV) [L, H, d] in float64, equal to ``attention_backward`` of
    the whole sequence."""
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(do)
    L, H, d = Q.shape
    parts_of = _ring_parts(L, world, layout)
    O, LSE = ring_attention_forward(Q, K, V, scale, causal, world, layout)
    D = (dO * O).sum(axis=-1)                                  # [L, H]
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for r in range(world):
        for t in range(world):
            s_ = (r - t) % world
            for qi, ki, diag in ring_blocks(r, t, world, causal, layout):
                rows, cols = slice(*parts_of[r][qi]), slice(*parts_of[s_][ki])
                for h in range(H):
                    Qr, Ks, Vs, dOr = Q[rows, h], K[cols, h], V[cols, h], dO[rows, h]
                    P = np.exp((Qr @ Ks.T) * scale - LSE[rows, h][:, None])
                    if diag:
                        P[np.triu_indices(P.shape[0], k=1)] = 0.0
                    dS = P * (dOr @ Vs.T - D[rows, h][:, None])
                    dQ[rows, h] += scale * (dS @ Ks)
                    dK[cols, h] += scale * (dS.T @ Qr)
                    dV[cols, h] += P.T @ dOr
    return dQ, dK, dV


# ----------------------------------------------------------------------------- dropout on P


_PHILOX_M = (0xD2511F53, 0xCD9E8D57)   # round multipliers
_PHILOX_W = (0x9E3779B9, 0xBB67AE85)   # key schedule (Weyl) increments
_U32 = 0xFFFFFFFF


def philox4x32_10(counter, key):
    """Philox4x32 with 10 rounds (Salmon, Moraes, Dror, Shaw: "Parallel random numbers: as easy as
    1, 2, 3", SC 2011): a counter-based generator mapping a 128-bit counter and a 64-bit key to 128
    random bits.  ``counter`` is 4 arrays (or ints) of uint32 words, ``key`` 2; broadcasting numpy
    arrays are processed element-wise.  Each round multiplies words 0 and 2 by fixed constants
    (full 64-bit products), and mixes the high halves with words 1, 3 and the round key; the key
    is bumped by fixed increments between rounds."""
    c = [np.asarray(x, dtype=np.uint64) & _U32 for x in counter]
    k0 = np.asarray(key[0], dtype=np.uint64) & _U32
    k1 = np.asarray(key[1], dtype=np.uint64) & _U32
    for r in range(10):
        if r > 0:
            k0 = (k0 + _PHILOX_W[0]) & _U32
            k1 = (k1 + _PHILOX_W[1]) & _U32
        p0 = c[0] * np.uint64(_PHILOX_M[0])
        p1 = c[2] * np.uint64(_PHILOX_M[1])
        hi0, lo0 = p0 >> np.uint64(32), p0 & _U32
        hi1, lo1 = p1 >> np.uint64(32), p1 & _U32
        c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return [x.astype(np.uint64) for x in c]


def dropout_threshold(p: float) -> int:
    """Dropout decisions compare one random byte with t = round(256·p) (clamped to 0…255): the
    element is kept when byte ≥ t, so the drop probability is t/256 and kept elements are scaled
    by 256/(256 − t) (inverted dropout, the expectation of P unchanged)."""
    if not (0.0 <= p < 1.0):
        raise ValueError("dropout probability must be in [0, 1)")
    return min(255, int(math.floor(p * 256.0 + 0.5)))


def dropout_keep_mask(L: int, bh: int, seed: int, offset: int, t: int) -> np.ndarray:
    """Keep mask [L, L] (query i, key j, positions inside one sequence) of the (sequence, head)
    with global index bh = b·H + h.  One Philox call covers a 4×4 block: counter = (j / 4, i / 4,
    bh, offset), key = the two 32-bit halves of ``seed``; element (i, j) uses byte j mod 4 of
    output word i mod 4."""
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    words = philox4x32_10([j >> 2, i >> 2, np.full((1, 1), bh), np.full((1, 1), offset)],
                          [seed & _U32, (seed >> 32) & _U32])
    w = np.select([(i & 3) == r for r in range(4)], [np.broadcast_to(x, (L, L)) for x in words])
    byte = (w >> (8 * (j & 3)).astype(np.uint64)) & np.uint64(0xFF)
    return byte >= t


def attention_forward_dropout(q, k, v, scale: float, causal: bool, dropout_p: float, seed: int, offset: int = 0,
                              cu_seqlens=None, B: Optional[int] = None, N: Optional[int] = None):
    """O = dropout(P) V with the keep mask of ``dropout_keep_mask``; LSE is that of the undropped
    softmax (the statistic the backward needs to recompute P).  Dropout on the probabilities is
    the ``dropout_p`` of the scaled-dot-product-attention interface (Flash Attention 优化, SDPA
    signature)."""
    Q, K, V = _f64(q), _f64(k), _f64(v)
    T, H, d = Q.shape
    t = dropout_threshold(dropout_p)
    keep_scale = 256.0 / (256.0 - t)
    if cu_seqlens is not None:
        B = len(np.asarray(cu_seqlens).reshape(-1)) - 1
    elif B is None:
        B = 1
    segs = sequence_segments(T, B, T // B if N is None else N, cu_seqlens)
    O = np.zeros((T, H, d))
    LSE = np.full((T, H), -np.inf)
    for b, (lo, L) in enumerate(segs):
        hi = lo + L
        for h in range(H):
            if L == 0:
                continue
            S = _scores(Q[lo:hi, h], K[lo:hi, h], scale, causal)
            P, m, ell = _softmax_rows(S)
            M = dropout_keep_mask(hi - lo, b * H + h, seed, offset, t)
            O[lo:hi, h] = (P * M * keep_scale) @ V[lo:hi, h]
            LSE[lo:hi, h] = m + np.log(ell)
    return O, LSE


def attention_backward_dropout(q, k, v, do, scale: float, causal: bool, dropout_p: float, seed: int,
                               offset: int = 0, cu_seqlens=None, B: Optional[int] = None, N: Optional[int] = None):
    """Gradients of ``attention_forward_dropout`` (the keep mask is a constant of the call): with
    Z = M·s/(1 − p)·P, O = Z V:  dV = Zᵀ dO,  dP = (dO Vᵀ) ∘ M·s,  D_i = Σ_j P_ij dP_ij
    (= Σ_c dO_ic O_ic),  dS = P ∘ (dP − D),  dQ = scale·dS K,  dK = scale·dSᵀ Q."""
    Q, K, V, dO = _f64(q), _f64(k), _f64(v), _f64(do)
    T, H, d = Q.shape
    t = dropout_threshold(dropout_p)
    keep_scale = 256.0 / (256.0 - t)
    if cu_seqlens is not None:
        B = len(np.asarray(cu_seqlens).reshape(-1)) - 1
    elif B is None:
        B = 1
    segs = sequence_segments(T, B, T // B if N is None else N, cu_seqlens)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b, (lo, L) in enumerate(segs):
        hi = lo + L
        for h in range(H):
            if L == 0:
                continue
            S = _scores(Q[lo:hi, h], K[lo:hi, h], scale, causal)
            P, _, _ = _softmax_rows(S)
            Mk = dropout_keep_mask(hi - lo, b * H + h, seed, offset, t) * keep_scale
            dV[lo:hi, h] = (P * Mk).T @ dO[lo:hi, h]
            dP = (dO[lo:hi, h] @ V[lo:hi, h].T) * Mk
            Dv = (P * dP).sum(axis=1)
            dS = P * (dP - Dv[:, None])
            dQ[lo:hi, h] = scale * dS @ K[lo:hi, h]
            dK[lo:hi, h] = scale * dS.T @ Q[lo:hi, h]
    return dQ, dK, dV
