"""Pins for the fp64 oracle: what the pages and the mathematics fix, not the oracle itself.

Each test checks the oracle against something other than its own formula:
the worked examples printed on the pages (``tests/golden/``), closed forms,
invariants that a wrong term, sign, index or operand order would break,
brute force (the tiled recurrence of the pages on tiny inputs) and central
finite differences for the backward.  ``test_pins_catch_planted_mistakes``
plants plausible mistakes in a copy of the oracle and checks that the pins
reject every one of them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _hand_qkv(d=4):
    """The narration's example: scale·q·k_j = ln c_j, V_j = value_j (feature 0)."""
    ex = _load("hand_example.json")
    scale = 0.5
    q = np.zeros((4, 1, d))
    k = np.zeros((4, 1, d))
    v = np.zeros((4, 1, d))
    q[:, 0, 0] = 1.0 / scale
    k[:, 0, 0] = np.log(ex["exp_scores"])
    v[:, 0, 0] = ex["v"]
    return ex, q, k, v, scale


def _rand(rng, T, H, d):
    return rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d)), rng.standard_normal((T, H, d))


# ----------------------------------------------------------------------------- worked examples


def test_hand_example_one_shot():
    ex, q, k, v, scale = _hand_qkv()
    O, LSE = oracle.attention_forward(q, k, v, scale, causal=False)
    assert np.all(np.abs(O[:, 0, 0] - ex["full"]["result"]) < 1e-12)
    # LSE = ln(sum of exponentiated scores) = ln(weight total)
    assert np.all(np.abs(np.exp(LSE[:, 0]) - ex["full"]["weight_total"]) < 1e-12)
    # weighted sum = result x weight total
    assert abs(O[0, 0, 0] * np.exp(LSE[0, 0]) - ex["full"]["weighted_sum"]) < 1e-10
    assert np.all(O[:, 0, 1:] == 0.0)


def test_hand_example_two_blocks_trace():
    ex, q, k, v, scale = _hand_qkv()
    trace = []
    O, _ = oracle.online_blockwise_forward(q[:1, 0], k[:, 0], v[:, 0], scale, bq=1, bk=2, trace=trace)
    assert len(trace) == 2
    _, _, m1, l1, num1 = trace[0]
    _, _, m2, l2, num2 = trace[1]
    b1, b2 = ex["after_block_1"], ex["after_block_2"]
    assert abs(math.exp(m1[0]) - b1["max_exp_score"]) < 1e-12
    assert abs(l1[0] - b1["denominator"]) < 1e-12
    assert abs(num1[0, 0] - b1["numerator"]) < 1e-12
    assert abs(math.exp(m1[0] - m2[0]) - ex["rescale_factor_at_block_2"]) < 1e-12
    assert abs(l2[0] - b2["denominator"]) < 1e-12
    assert abs(num2[0, 0] - b2["numerator"]) < 1e-12
    assert abs(O[0, 0] - b2["result"]) < 1e-12
    # the block-2 weights: new denominator minus the rescaled old one, and each weight
    new_part = l2[0] - b1["denominator"] * ex["rescale_factor_at_block_2"]
    assert abs(new_part - sum(ex["block_2_weights"])) < 1e-12


def test_hand_example_causal_prefixes():
    """Causal version of the same row set: row i averages the first i+1 values."""
    ex, q, k, v, scale = _hand_qkv()
    O, LSE = oracle.attention_forward(q, k, v, scale, causal=True)
    c = np.array(ex["exp_scores"], float)
    vals = np.array(ex["v"], float)
    for i in range(4):
        want = (c[: i + 1] * vals[: i + 1]).sum() / c[: i + 1].sum()
        assert abs(O[i, 0, 0] - want) < 1e-12
        assert abs(LSE[i, 0] - math.log(c[: i + 1].sum())) < 1e-12
    assert abs(O[1, 0, 0] - 50.0 / 3.0) < 1e-12 and abs(O[2, 0, 0] - 170.0 / 7.0) < 1e-12


def test_online_softmax_numeric_example():
    ex = _load("online_softmax_example.json")
    stats = oracle.online_softmax_stats(ex["x"], ex["blocks"])
    (m1, l1), (m2, l2) = stats
    assert m1 == ex["block_1"]["m"] and m2 == ex["block_2"]["m"]
    # printed to 4 decimals, with the page summing already-rounded parts
    assert abs(l1 - ex["block_1"]["l"]) < 1e-4
    assert abs(l2 - ex["block_2"]["l"]) < 2e-4
    assert abs(l1 * math.exp(m1 - m2) - ex["block_2"]["rescaled_old_l"]) < 2e-4
    # the merge form (two partial pairs) gives the same statistics
    mm, lm = oracle.merge_softmax_stats(m1, l1, 4.0, ex["block_2"]["new_block_contribution"])
    assert mm == 4.0 and abs(lm - ex["block_2"]["l"]) < 2e-4
    # one-shot softmax through the attention oracle: q·k_j = x_j, V = identity rows
    x = np.array(ex["x"], float)
    q = np.zeros((1, 1, 4)); q[0, 0, 0] = 1.0
    k = np.zeros((4, 1, 4)); k[:, 0, 0] = x
    v = np.eye(4)[:, None, :]
    # one query attending to four keys: put the query last in a causal-free 4-token call
    Q = np.zeros((4, 1, 4)); Q[:] = q
    O, LSE = oracle.attention_forward(Q, k, v, 1.0)
    assert np.allclose(O[0, 0], ex["one_shot"]["softmax"], atol=5e-4)
    assert abs(math.exp(LSE[0, 0] - ex["one_shot"]["max"]) - ex["one_shot"]["sum"]) < 5e-4
    assert np.allclose(np.exp(x - x.max()), ex["one_shot"]["exp"], atol=5e-5)


# ----------------------------------------------------------------------------- closed forms and invariants


@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 37, 3, 8)
    v[:] = 1.0  # O = P·1 = row sums of P
    O, _ = oracle.attention_forward(q, k, v, 0.7, causal=causal)
    assert np.max(np.abs(O - 1.0)) < 1e-12


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(causal):
    """Adding u to every key adds scale·q_i·u to row i of S: P and O unchanged, LSE shifted."""
    rng = np.random.default_rng(2)
    q, k, v = _rand(rng, 29, 2, 16)
    u = rng.standard_normal(16) * 3.0
    scale = 0.25
    O1, L1 = oracle.attention_forward(q, k, v, scale, causal=causal)
    O2, L2 = oracle.attention_forward(q, k + u, v, scale, causal=causal)
    assert np.max(np.abs(O1 - O2)) < 1e-11
    assert np.max(np.abs((L2 - L1) - scale * np.einsum("thd,d->th", q, u))) < 1e-10


def test_large_scores_do_not_overflow():
    """The row max is subtracted before exponentiating (safe softmax)."""
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 16, 1, 4)
    O1, L1 = oracle.attention_forward(q, k, v, 1.0)
    big = np.zeros(4); big[0] = 1.0
    # add 1000 to every score of every row through a key shift along q's direction
    q2 = np.concatenate([q, np.ones((16, 1, 1))], axis=2)
    k2 = np.concatenate([k, np.full((16, 1, 1), 1000.0)], axis=2)
    v2 = np.concatenate([v, np.zeros((16, 1, 1))], axis=2)
    O2, L2 = oracle.attention_forward(q2, k2, v2, 1.0)
    assert np.all(np.isfinite(O2)) and np.max(np.abs(O2[..., :4] - O1)) < 1e-10
    assert np.max(np.abs(L2 - (L1 + 1000.0))) < 1e-9


@pytest.mark.parametrize("causal", [False, True])
def test_uniform_keys_give_mean_of_values(causal):
    rng = np.random.default_rng(4)
    L, d = 11, 6
    q = rng.standard_normal((L, 1, d))
    k = np.tile(rng.standard_normal((1, 1, d)), (L, 1, 1))
    v = rng.standard_normal((L, 1, d))
    scale = 0.3
    O, LSE = oracle.attention_forward(q, k, v, scale, causal=causal)
    for i in range(L):
        n = i + 1 if causal else L
        assert np.max(np.abs(O[i, 0] - v[:n, 0].mean(axis=0))) < 1e-12
        s = scale * float(q[i, 0] @ k[0, 0])
        assert abs(LSE[i, 0] - (s + math.log(n))) < 1e-12


def test_single_token_returns_its_value():
    rng = np.random.default_rng(5)
    q, k, v = _rand(rng, 1, 3, 5)
    O, LSE = oracle.attention_forward(q, k, v, 0.4, causal=True)
    assert np.max(np.abs(O - v)) < 1e-15
    assert np.max(np.abs(LSE - 0.4 * np.einsum("thd,thd->th", q, k))) < 1e-14


def test_causal_row_ignores_future_keys():
    """Changing keys/values after position i leaves causal row i unchanged."""
    rng = np.random.default_rng(6)
    q, k, v = _rand(rng, 20, 2, 4)
    O1, L1 = oracle.attention_forward(q, k, v, 0.5, causal=True)
    k2, v2 = k.copy(), v.copy()
    k2[12:] = rng.standard_normal(k2[12:].shape) * 10
    v2[12:] = rng.standard_normal(v2[12:].shape) * 10
    O2, L2 = oracle.attention_forward(q, k2, v2, 0.5, causal=True)
    assert np.array_equal(O1[:12], O2[:12]) and np.array_equal(L1[:12], L2[:12])
    assert np.max(np.abs(O1[12:] - O2[12:])) > 1e-3


def test_key_permutation_invariance_non_causal():
    rng = np.random.default_rng(7)
    q, k, v = _rand(rng, 17, 2, 8)
    perm = rng.permutation(17)
    O1, L1 = oracle.attention_forward(q, k, v, 0.35)
    O2, L2 = oracle.attention_forward(q, k[perm], v[perm], 0.35)
    assert np.max(np.abs(O1 - O2)) < 1e-12 and np.max(np.abs(L1 - L2)) < 1e-12


def test_brute_force_scalar_loop_tiny():
    """Direct scalar loops (no matrix products) on a 3-token, 2-feature case."""
    rng = np.random.default_rng(8)
    q, k, v = _rand(rng, 3, 1, 2)
    scale = 0.9
    for causal in (False, True):
        O, LSE = oracle.attention_forward(q, k, v, scale, causal=causal)
        for i in range(3):
            js = range(i + 1) if causal else range(3)
            s = {j: scale * (q[i, 0, 0] * k[j, 0, 0] + q[i, 0, 1] * k[j, 0, 1]) for j in js}
            z = sum(math.exp(x) for x in s.values())
            for c in range(2):
                want = sum(math.exp(s[j]) * v[j, 0, c] for j in js) / z
                assert abs(O[i, 0, c] - want) < 1e-12
            assert abs(LSE[i, 0] - math.log(z)) < 1e-12


# ----------------------------------------------------------------------------- tiled recurrence


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bq,bk", [(1, 1), (64, 64), (3, 5), (7, 2), (16, 13), (50, 50)])
def test_blockwise_recurrence_equals_one_shot(causal, bq, bk):
    rng = np.random.default_rng(100 + bq * 7 + bk)
    q, k, v = _rand(rng, 50, 2, 8)
    scale = 1.0 / math.sqrt(8)
    O1, L1 = oracle.attention_forward(q, k, v, scale, causal=causal)
    O2, L2 = oracle.online_blockwise_forward(q, k, v, scale, causal=causal, bq=bq, bk=bk)
    assert np.max(np.abs(O1 - O2)) < 1e-12
    assert np.max(np.abs(L1 - L2)) < 1e-12


def test_online_stats_random_splits_match_one_shot():
    rng = np.random.default_rng(9)
    for _ in range(50):
        n = int(rng.integers(1, 40))
        x = rng.standard_normal(n) * 5
        cuts = sorted(set(int(c) for c in rng.integers(1, n + 1, size=int(rng.integers(0, 5)))) | {n})
        blocks = [b - a for a, b in zip([0] + cuts[:-1], cuts)]
        m, l = oracle.online_softmax_stats(x, blocks)[-1]
        assert m == x.max()
        assert abs(l - np.exp(x - x.max()).sum()) < 1e-12


# ----------------------------------------------------------------------------- varlen and row sampling


def test_varlen_equals_separate_sequences():
    rng = np.random.default_rng(10)
    lens = [5, 1, 9, 0, 4]
    cu = np.cumsum([0] + lens)
    T = int(cu[-1])
    q, k, v = _rand(rng, T, 2, 4)
    do = rng.standard_normal((T, 2, 4))
    for causal in (False, True):
        O, L = oracle.attention_forward(q, k, v, 0.6, causal, cu_seqlens=cu)
        dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.6, causal, cu_seqlens=cu)
        for b, n in enumerate(lens):
            if n == 0:
                continue
            sl = slice(cu[b], cu[b + 1])
            Ob, Lb = oracle.attention_forward(q[sl], k[sl], v[sl], 0.6, causal)
            g = oracle.attention_backward(q[sl], k[sl], v[sl], do[sl], 0.6, causal)
            assert np.array_equal(O[sl], Ob) and np.array_equal(L[sl], Lb)
            for a, bb in zip((dq, dk, dv), g):
                assert np.array_equal(a[sl], bb)


def test_rows_sampler_matches_full():
    rng = np.random.default_rng(11)
    lens = [7, 12, 3]
    cu = np.cumsum([0] + lens)
    q, k, v = _rand(rng, int(cu[-1]), 3, 4)
    rows = list(range(int(cu[-1])))
    for causal in (False, True):
        O, L = oracle.attention_forward(q, k, v, 0.5, causal, cu_seqlens=cu)
        Or, Lr = oracle.attention_forward_rows(q, k, v, rows, 0.5, causal, cu_seqlens=cu)
        assert np.max(np.abs(O - Or)) < 1e-12 and np.max(np.abs(L - Lr)) < 1e-12


def test_row_block_fwd_bwd_sums_to_full():
    rng = np.random.default_rng(12)
    L, H, d = 24, 2, 4
    q, k, v = _rand(rng, L, H, d)
    do = rng.standard_normal((L, H, d))
    for causal in (False, True):
        O, LSE = oracle.attention_forward(q, k, v, 0.5, causal)
        dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, causal)
        for h in range(H):
            dk_sum = np.zeros((L, d)); dv_sum = np.zeros((L, d))
            for lo in range(0, L, 10):
                hi = min(lo + 10, L)
                o, lse, dqr, dkr, dvr = oracle.attention_fwd_bwd_rows(q, k, v, do, lo, hi, 0.5, causal, head=h)
                assert np.max(np.abs(o - O[lo:hi, h])) < 1e-12
                assert np.max(np.abs(lse - LSE[lo:hi, h])) < 1e-12
                assert np.max(np.abs(dqr - dq[lo:hi, h])) < 1e-12
                dk_sum += dkr; dv_sum += dvr
            assert np.max(np.abs(dk_sum - dk[:, h])) < 1e-12
            assert np.max(np.abs(dv_sum - dv[:, h])) < 1e-12


# ----------------------------------------------------------------------------- backward


def _fd_check(q, k, v, do, scale, causal, cu=None, h=1e-6):
    dq, dk, dv = oracle.attention_backward(q, k, v, do, scale, causal, cu_seqlens=cu)

    def f(qq, kk, vv):
        O, _ = oracle.attention_forward(qq, kk, vv, scale, causal, cu_seqlens=cu)
        return float((O * do).sum())

    worst = 0.0
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        it = np.nditer(grad, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            args_p = [q.copy(), k.copy(), v.copy()]
            args_m = [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            fd = (f(*args_p) - f(*args_m)) / (2 * h)
            worst = max(worst, abs(fd - grad[idx]) / max(1.0, abs(grad[idx])))
    return worst


@pytest.mark.parametrize("causal", [False, True])
def test_backward_finite_differences(causal):
    rng = np.random.default_rng(13)
    q, k, v = _rand(rng, 6, 2, 3)
    do = rng.standard_normal((6, 2, 3))
    assert _fd_check(q, k, v, do, 0.8, causal) < 1e-6


def test_backward_finite_differences_varlen():
    rng = np.random.default_rng(14)
    cu = np.array([0, 3, 4, 8])
    q, k, v = _rand(rng, 8, 1, 2)
    do = rng.standard_normal((8, 1, 2))
    assert _fd_check(q, k, v, do, 1.1, True, cu=cu) < 1e-6


@pytest.mark.parametrize("causal", [False, True])
def test_backward_sum_invariants(causal):
    """Σ_j dK_j = 0 (softmax is shift invariant in the keys) and Σ_j dV_j = Σ_i dO_i."""
    rng = np.random.default_rng(15)
    q, k, v = _rand(rng, 33, 3, 8)
    do = rng.standard_normal((33, 3, 8))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.4, causal)
    assert np.max(np.abs(dk.sum(axis=0))) < 1e-10
    assert np.max(np.abs(dv.sum(axis=0) - do.sum(axis=0))) < 1e-10


def test_backward_uniform_keys_closed_form():
    """With all keys equal P is uniform and dV_j = (1/L)·Σ_i dO_i (non-causal)."""
    rng = np.random.default_rng(16)
    L, d = 9, 4
    q = rng.standard_normal((L, 1, d))
    k = np.tile(rng.standard_normal((1, 1, d)), (L, 1, 1))
    v = rng.standard_normal((L, 1, d))
    do = rng.standard_normal((L, 1, d))
    dq, dk, dv = oracle.attention_backward(q, k, v, do, 0.5, False)
    for j in range(L):
        assert np.max(np.abs(dv[j, 0] - do[:, 0].mean(axis=0))) < 1e-12
    # dQ_i = scale · Σ_j P_ij (dP_ij − D_i) k_j = scale · k · Σ_j P_ij (dP_ij − D_i) = 0
    assert np.max(np.abs(dq)) < 1e-12


def test_flop_convention():
    # 4·B·h·s²·d for B=4, h=16, s=8192, d=128, halved when causal
    assert oracle.attention_flops([8192] * 4, 16, 128, causal=False) == 4 * 4 * 16 * 8192 ** 2 * 128
    assert oracle.attention_flops([8192] * 4, 16, 128, causal=True) == 2 * 4 * 16 * 8192 ** 2 * 128
    assert oracle.attention_flops([10], 1, 2, causal=False, backward=True) == 2.5 * 4 * 100 * 2


# ----------------------------------------------------------------------------- planted mistakes


def _pins_pass():
    """A compact battery of the pins above; returns False as soon as one fails."""
    checks = [
        test_hand_example_one_shot, test_hand_example_causal_prefixes,
        lambda: test_rows_of_p_sum_to_one(True), lambda: test_shift_invariance(True),
        test_large_scores_do_not_overflow, lambda: test_uniform_keys_give_mean_of_values(True),
        test_brute_force_scalar_loop_tiny, test_causal_row_ignores_future_keys,
        lambda: test_backward_finite_differences(True), lambda: test_backward_sum_invariants(True),
        test_backward_uniform_keys_closed_form,
    ]
    for c in checks:
        try:
            with np.errstate(all="ignore"):
                c()
        except (AssertionError, FloatingPointError, ValueError, IndexError):
            return False
    return True


def test_pins_catch_planted_mistakes(monkeypatch):
    assert _pins_pass()
    orig_scores, orig_softmax = A._scores, A._softmax_rows

    def no_scale(Q, K, scale, causal):
        return orig_scores(Q, K, 1.0, causal)

    def transposed(Q, K, scale, causal):
        S = (K @ Q.T) * scale if Q.shape[0] == K.shape[0] else (Q @ K.T) * scale
        if causal:
            S[np.triu_indices(S.shape[0], k=1)] = -np.inf
        return S

    def upper_mask(Q, K, scale, causal):
        S = (Q @ K.T) * scale
        if causal:
            S[np.tril_indices(S.shape[0], k=-1)] = -np.inf
        return S

    def mask_off_by_one(Q, K, scale, causal):
        S = (Q @ K.T) * scale
        if causal:
            S[np.triu_indices(S.shape[0], k=2)] = -np.inf
        return S

    def no_max_shift(S):
        E = np.exp(S)
        ell = E.sum(axis=1)
        return E / ell[:, None], np.zeros(S.shape[0]), ell

    def wrong_sign(S):
        m = S.max(axis=1)
        E = np.exp(m[:, None] - S)
        ell = E.sum(axis=1)
        return E / ell[:, None], m, ell

    def dropped_norm(S):
        m = S.max(axis=1)
        E = np.exp(S - m[:, None])
        return E, m, E.sum(axis=1)

    for name, patch in [("_scores", no_scale), ("_scores", transposed), ("_scores", upper_mask),
                        ("_scores", mask_off_by_one), ("_softmax_rows", no_max_shift),
                        ("_softmax_rows", wrong_sign), ("_softmax_rows", dropped_norm)]:
        with monkeypatch.context() as mp:
            mp.setattr(A, name, patch)
            assert not _pins_pass(), f"planted mistake {patch.__name__} was not caught"

    # a mistake in the backward only: D computed without P, dK missing its scale
    orig_bwd = A.attention_backward

    def bwd_no_dk_scale(q, k, v, do, scale, causal=False, cu_seqlens=None, B=None, N=None):
        dq, dk, dv = orig_bwd(q, k, v, do, scale, causal, cu_seqlens, B, N)
        return dq, dk / scale, dv

    with monkeypatch.context() as mp:
        mp.setattr(A, "attention_backward", bwd_no_dk_scale)
        mp.setattr(oracle, "attention_backward", bwd_no_dk_scale)
        assert not _pins_pass()


# ----------------------------------------------------------------------------- decode (one query per sequence)


def _decode_pins_pass(decode, split=None):
    """The decode pins, run against a given implementation (the oracle's, or a planted mistake)."""
    try:
        # the hand example: the one query row scores ln c_j against the four keys → O = 29, LSE = ln 10
        ex, q, k, v, scale = _hand_qkv()
        O, L = decode(q[:1, :, :], k, v, scale, B=1, Nk=4)
        assert abs(O[0, 0, 0] - ex["full"]["result"]) < 1e-12
        assert abs(L[0, 0] - math.log(ex["full"]["weight_total"])) < 1e-12
        # the last row of causal self-attention (pinned above) is a decode step of the last token
        rng = np.random.default_rng(7)
        for Lk in (1, 5, 17):
            Q, K, V = _rand(rng, Lk, 2, 4)
            O_ref, L_ref = oracle.attention_forward(Q * 3.0, K, V, 0.37, causal=True)
            O, L = decode(Q[Lk - 1:] * 3.0, K, V, 0.37, B=1, Nk=Lk)
            assert np.abs(O[0] - O_ref[Lk - 1]).max() < 1e-12 and np.abs(L[0] - L_ref[Lk - 1]).max() < 1e-12
        # brute force with scalar loops on a tiny packed batch, one sequence empty
        q = rng.standard_normal((3, 1, 3))
        k = rng.standard_normal((6, 1, 3))
        v = rng.standard_normal((6, 1, 3))
        cu = [0, 4, 4, 6]
        O, L = decode(q, k, v, 0.8, cu_seqlens_k=cu)
        for b in range(3):
            lo, hi = cu[b], cu[b + 1]
            if hi == lo:
                assert np.all(O[b] == 0.0) and L[b, 0] == -math.inf
                continue
            w = [math.exp(0.8 * sum(q[b, 0, c] * k[j, 0, c] for c in range(3))) for j in range(lo, hi)]
            tot = sum(w)
            for c in range(3):
                assert abs(O[b, 0, c] - sum(w[j - lo] * v[j, 0, c] for j in range(lo, hi)) / tot) < 1e-12
            assert abs(L[b, 0] - math.log(tot)) < 1e-12
        # large scores must not overflow (the max is subtracted first): every score is about 2400
        q = np.full((1, 1, 2), 40.0)
        k = 30.0 + rng.standard_normal((8, 1, 2))
        v = rng.standard_normal((8, 1, 2))
        O, L = decode(q, k, v, 1.0, B=1, Nk=8)
        assert np.all(np.isfinite(O)) and np.isfinite(L[0, 0])
        if split is not None:
            q = rng.standard_normal((4, 3, 8))
            k = rng.standard_normal((50, 3, 8))
            v = rng.standard_normal((50, 3, 8))
            cu = [0, 20, 20, 33, 50]
            O_ref, L_ref = decode(q, k, v, 0.5, cu_seqlens_k=cu)
            for chunk in (1, 2, 3, 7, 16, 20, 64):
                O, L = split(q, k, v, 0.5, chunk, cu_seqlens_k=cu)
                assert np.abs(O - O_ref).max() < 1e-12
                fin = np.isfinite(L_ref)
                assert np.all(fin == np.isfinite(L)) and np.abs(L[fin] - L_ref[fin]).max() < 1e-12
        return True
    except (AssertionError, FloatingPointError, ValueError, IndexError):
        return False


def test_decode_oracle_pins():
    assert _decode_pins_pass(oracle.decode_forward, oracle.split_kv_decode)


def test_split_kv_chunk_of_one_is_the_per_element_recurrence():
    """With one key per chunk, the merged (m, ℓ) after each key are the page's running statistics."""
    rng = np.random.default_rng(11)
    q = rng.standard_normal((1, 1, 4))
    k = rng.standard_normal((9, 1, 4))
    v = rng.standard_normal((9, 1, 4))
    scores = [0.5 * float(k[j, 0] @ q[0, 0]) for j in range(9)]
    _, _, parts = oracle.split_kv_decode(q, k, v, 0.5, 1, B=1, Nk=9, return_partials=True)
    stats = oracle.online_softmax_stats(scores, [1] * 9)
    m, ell = -math.inf, 0.0
    for j, ((m_c, l_c, O_c), (m_ref, l_ref)) in enumerate(zip(parts[0], stats)):
        # one key: its own score is the max, the sum is e^0 = 1 and the partial output is that key's value
        assert m_c == pytest.approx(scores[j], abs=1e-15) and l_c == 1.0
        assert np.array_equal(O_c, v[j, 0])
        m, ell = oracle.merge_softmax_stats(m, ell, m_c, l_c)
        assert m == pytest.approx(m_ref, abs=1e-15) and ell == pytest.approx(l_ref, rel=1e-14)


def test_decode_pins_catch_planted_mistakes():
    def no_scale(q, k, v, scale, cu_seqlens_k=None, B=None, Nk=None):
        return oracle.decode_forward(q, k, v, 1.0, cu_seqlens_k, B, Nk)

    def no_max_shift(q, k, v, scale, cu_seqlens_k=None, B=None, Nk=None):
        Q, K, V = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
        segs = A._key_segments(K.shape[0], Q.shape[0] if B is None else B, Nk, cu_seqlens_k)
        O = np.zeros(Q.shape)
        L = np.full(Q.shape[:2], -np.inf)
        with np.errstate(over="raise"):
            for b, (lo, hi) in enumerate(segs):
                for h in range(Q.shape[1]):
                    if hi > lo:
                        e = np.exp((K[lo:hi, h] @ Q[b, h]) * scale)
                        O[b, h] = e @ V[lo:hi, h] / e.sum()
                        L[b, h] = math.log(e.sum())
        return O, L

    def drops_last_key(q, k, v, scale, cu_seqlens_k=None, B=None, Nk=None):
        segs = A._key_segments(np.asarray(k).shape[0], np.asarray(q).shape[0] if B is None else B, Nk, cu_seqlens_k)
        rows = [j for lo, hi in segs for j in range(lo, max(lo, hi - 1))]
        cu = np.cumsum([0] + [max(0, hi - lo - 1) for lo, hi in segs])
        return oracle.decode_forward(q, np.asarray(k)[rows], np.asarray(v)[rows], scale, cu_seqlens_k=cu)

    def wrong_merge_sign(q, k, v, scale, chunk, cu_seqlens_k=None, B=None, Nk=None):
        O, L, parts = oracle.split_kv_decode(q, k, v, scale, chunk, cu_seqlens_k, B, Nk, return_partials=True)
        Ob = np.zeros_like(O)
        for idx, ps in enumerate(parts):
            b, h = divmod(idx, O.shape[1])
            if not ps:
                continue
            m = max(p[0] for p in ps)
            ell = sum(p[1] * math.exp(m - p[0]) for p in ps)   # the sign of the exponent flipped
            Ob[b, h] = sum(p[2] * math.exp(m - p[0]) for p in ps) / ell
        return Ob, L

    assert not _decode_pins_pass(no_scale)
    assert not _decode_pins_pass(no_max_shift)
    assert not _decode_pins_pass(drops_last_key)
    assert not _decode_pins_pass(oracle.decode_forward, wrong_merge_sign)


# ----------------------------------------------------------------------------- dropout on P


def test_philox_known_answers():
    kat = _load("philox4x32_10_kat.json")
    for vec in kat["vectors"]:
        ctr = [int(x, 16) for x in vec["counter"]]
        key = [int(x, 16) for x in vec["key"]]
        got = [int(x) for x in oracle.philox4x32_10(ctr, key)]
        assert got == [int(x, 16) for x in vec["output"]]


def test_dropout_mask_mapping_scalar():
    """Element (i, j): byte j mod 4 of word i mod 4 of Philox(counter (j/4, i/4, bh, offset), seed)."""
    seed, bh, off, t = 0x1234_5678_9ABC_DEF0, 5, 3, 77
    M = oracle.dropout_keep_mask(23, bh, seed, off, t)
    for i in range(23):
        for j in range(23):
            w = [int(x) for x in oracle.philox4x32_10([j >> 2, i >> 2, bh, off], [seed & 0xFFFFFFFF, seed >> 32])]
            byte = (w[i & 3] >> (8 * (j & 3))) & 0xFF
            assert bool(M[i, j]) == (byte >= t)


@pytest.mark.parametrize("p", [0.0, 0.1, 0.5, 0.9])
def test_dropout_keep_fraction(p):
    t = oracle.dropout_threshold(p)
    M = oracle.dropout_keep_mask(512, 7, 99, 0, t)
    keep = 1.0 - t / 256.0
    n = M.size
    assert abs(M.mean() - keep) <= 5.0 * math.sqrt(keep * (1 - keep) / n) + 1e-12
    if p == 0.0:
        assert M.all()


def test_dropout_masks_differ_by_head_seed_offset():
    t = oracle.dropout_threshold(0.5)
    a = oracle.dropout_keep_mask(64, 0, 1, 0, t)
    for other in (oracle.dropout_keep_mask(64, 1, 1, 0, t), oracle.dropout_keep_mask(64, 0, 2, 0, t),
                  oracle.dropout_keep_mask(64, 0, 1, 1, t)):
        assert 0.3 < (a != other).mean() < 0.7


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_zero_is_plain_attention(causal):
    rng = np.random.default_rng(21)
    q, k, v = _rand(rng, 30, 2, 8)
    do = rng.standard_normal(q.shape)
    cu = [0, 13, 30]
    O1, L1 = oracle.attention_forward(q, k, v, 0.4, causal, cu_seqlens=cu)
    O2, L2 = oracle.attention_forward_dropout(q, k, v, 0.4, causal, 0.0, 5, cu_seqlens=cu)
    assert np.abs(O1 - O2).max() < 1e-12 and np.abs(L1 - L2).max() < 1e-12
    g1 = oracle.attention_backward(q, k, v, do, 0.4, causal, cu_seqlens=cu)
    g2 = oracle.attention_backward_dropout(q, k, v, do, 0.4, causal, 0.0, 5, cu_seqlens=cu)
    for a, b in zip(g1, g2):
        assert np.abs(a - b).max() < 1e-12


def test_dropout_is_unbiased_over_seeds():
    """Inverted dropout keeps the expectation: the mean of O over many seeds approaches the
    undropped O (a missing 1/(1 − p) would leave it short by the keep probability)."""
    rng = np.random.default_rng(3)
    q, k, v = _rand(rng, 16, 1, 4)
    O_ref, _ = oracle.attention_forward(q, k, v, 0.5, False)
    acc = np.zeros_like(O_ref)
    n = 400
    for s in range(n):
        acc += oracle.attention_forward_dropout(q, k, v, 0.5, False, 0.3, 1000 + s)[0]
    assert np.abs(acc / n - O_ref).max() < 0.06
    assert np.abs(acc / n * (1 - 77 / 256) - O_ref).max() > 0.05  # the unscaled mean would be visibly short


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_backward_finite_differences(causal):
    rng = np.random.default_rng(8 + int(causal))
    q, k, v = _rand(rng, 7, 1, 3)
    do = rng.standard_normal(q.shape)
    p, seed, scale = 0.3, 42, 0.7
    f = lambda q_, k_, v_: float((oracle.attention_forward_dropout(q_, k_, v_, scale, causal, p, seed)[0] * do).sum())
    dq, dk, dv = oracle.attention_backward_dropout(q, k, v, do, scale, causal, p, seed)
    h = 1e-6
    for arr, g in ((q, dq), (k, dk), (v, dv)):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            a1, a2 = arr.copy(), arr.copy()
            a1[idx] += h
            a2[idx] -= h
            args1 = [a1 if arr is x else x for x in (q, k, v)]
            args2 = [a2 if arr is x else x for x in (q, k, v)]
            num[idx] = (f(*args1) - f(*args2)) / (2 * h)
        assert np.linalg.norm(num - g) <= 1e-6 * max(1.0, np.linalg.norm(g))


def test_dropout_delta_identity():
    """D_i = Σ_j P_ij dP_ij equals Σ_c dO_ic O_ic also with dropout (O is the dropped output)."""
    rng = np.random.default_rng(4)
    q, k, v = _rand(rng, 20, 1, 5)
    do = rng.standard_normal(q.shape)
    p, seed, scale = 0.2, 7, 0.5
    O, _ = oracle.attention_forward_dropout(q, k, v, scale, True, p, seed)
    t = oracle.dropout_threshold(p)
    S = (q[:, 0] @ k[:, 0].T) * scale
    S[np.triu_indices(20, 1)] = -np.inf
    P = np.exp(S - S.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    dP = (do[:, 0] @ v[:, 0].T) * oracle.dropout_keep_mask(20, 0, seed, 0, t) * 256.0 / (256.0 - t)
    assert np.abs((P * dP).sum(axis=1) - (do[:, 0] * O[:, 0]).sum(axis=1)).max() < 1e-12


# ----------------------------------------------------------------------------- partial results: merge, ring schedule


def _empty_part(shape):
    return np.zeros(shape), np.full(shape[:-1], -np.inf)


def _ring_pins_pass(merge, ring):
    """The pins of merge_attention_partials and ring_attention_forward, run against a given pair of
    implementations (the oracle's, or planted mistakes)."""
    try:
        rng = np.random.default_rng(21)
        # (1) one query's partials over disjoint key sets (one of them empty) merge to its attention over
        # all keys, whatever the order of the parts
        q = rng.standard_normal((1, 2, 4))
        k = rng.standard_normal((11, 2, 4))
        v = rng.standard_normal((11, 2, 4))
        full = oracle.decode_forward(q, k, v, 0.7, B=1, Nk=11)
        sets = [[0, 3, 4], [], [1, 2, 5, 9], [6, 7, 8, 10]]
        parts = [oracle.decode_forward(q, k[idx], v[idx], 0.7, B=1, Nk=len(idx)) if idx else _empty_part((1, 2, 4))
                 for idx in sets]
        for order in (parts, parts[::-1], [parts[2], parts[0], parts[3], parts[1]]):
            O, L = merge(order)
            assert np.allclose(O, full[0], atol=1e-13, rtol=0) and np.allclose(L, full[1], atol=1e-13, rtol=0)
        # (2) one part comes back unchanged; an empty part changes nothing; two empty parts stay empty
        for ps in ([full], [full, _empty_part((1, 2, 4))], [_empty_part((1, 2, 4)), full]):
            O, L = merge(ps)
            assert np.array_equal(O, full[0]) and np.array_equal(L, full[1])
        O, L = merge([_empty_part((1, 2, 4)), _empty_part((1, 2, 4))])
        assert np.all(O == 0.0) and np.all(np.isneginf(L))
        # (3) log-sum-exps near 1000 (e^1000 overflows float64): shifting every part by 1000 shifts only LSE
        with np.errstate(over="raise", invalid="raise"):
            O, L = merge([(Ob, Lb + 1000.0) for Ob, Lb in parts])
        assert np.allclose(O, full[0], atol=1e-13, rtol=0) and np.allclose(L, full[1] + 1000.0, atol=1e-12, rtol=0)
        # (4) the ring schedule equals the definition for 1 … 6 ranks, causal and not
        qq, kk, vv = (rng.standard_normal((12, 2, 4)) for _ in range(3))
        for causal in (False, True):
            O_ref, L_ref = oracle.attention_forward(qq, kk, vv, 0.5, causal)
            for w in (1, 2, 3, 4, 6):
                O, L = ring(qq, kk, vv, 0.5, causal, w)
                assert np.allclose(O, O_ref, atol=1e-13, rtol=0) and np.allclose(L, L_ref, atol=1e-13, rtol=0)
        return True
    except (AssertionError, FloatingPointError):
        return False


def test_ring_and_merge_pins():
    assert _ring_pins_pass(oracle.merge_attention_partials, oracle.ring_attention_forward)


def test_ring_and_merge_pins_catch_planted_mistakes():
    merge, ring = oracle.merge_attention_partials, oracle.ring_attention_forward

    def merge_unshifted(ps):  # the weights e^{LSE_b} without the max shift
        O, L = (np.asarray(ps[0][0], dtype=np.float64), np.asarray(ps[0][1], dtype=np.float64))
        for Ob, Lb in ps[1:]:
            s = np.exp(L) + np.exp(Lb)
            O = (np.exp(L)[..., None] * O + np.exp(Lb)[..., None] * Ob) / s[..., None]
            L = np.log(s)
        return O, L

    def merge_swapped(ps):  # each part weighted by the other part's share
        O, L = ps[0]
        for Ob, Lb in ps[1:]:
            Ls = np.logaddexp(L, Lb)
            O = np.exp(Lb - Ls)[..., None] * O + np.exp(L - Ls)[..., None] * Ob
            L = Ls
        return O, L

    def merge_lse_max_only(ps):  # LSE taken as the larger part's, not the log of the sum
        O, L = merge(ps)
        return O, np.maximum.reduce([np.asarray(p[1]) for p in ps])

    def ring_variant(skip, diag_causal):
        def f(q, k, v, scale, causal, world):
            L_, H, d = q.shape
            S = L_ // world
            O, LSE = np.zeros((L_, H, d)), np.full((L_, H), -np.inf)
            for r in range(world):
                rows, parts = slice(r * S, (r + 1) * S), []
                for t in range(world):
                    s_ = (r - t) % world
                    if causal and skip(s_, r):
                        continue
                    cols = slice(s_ * S, (s_ + 1) * S)
                    parts.append(oracle.attention_forward(q[rows], k[cols], v[cols], scale,
                                                          causal and s_ == r and diag_causal))
                if parts:  # a rank whose every shard is skipped keeps O = 0, LSE = −∞
                    O[rows], LSE[rows] = merge(parts)
            return O, LSE
        return f

    ring_sees_future = ring_variant(lambda s_, r: False, True)     # later shards not skipped
    ring_skips_diagonal = ring_variant(lambda s_, r: s_ >= r, True)  # own shard skipped
    ring_diag_unmasked = ring_variant(lambda s_, r: s_ > r, False)  # diagonal block without its mask
    assert _ring_pins_pass(merge, ring_variant(lambda s_, r: s_ > r, True))  # the faithful restatement passes
    for m in (merge_unshifted, merge_swapped, merge_lse_max_only):
        assert not _ring_pins_pass(m, ring), m.__name__
    for rv in (ring_sees_future, ring_skips_diagonal, ring_diag_unmasked):
        assert not _ring_pins_pass(merge, rv)


def test_ring_backward_equals_definition():
    """The ring backward (blocks from the global LSE and D, dK/dV travelling with their shard) equals
    the whole-sequence backward for 1 … 6 ranks, causal and not; dropping the causal skip, using the
    block's own LSE instead of the global one, or leaving out D each breaks it."""
    rng = np.random.default_rng(33)
    q, k, v, do = (rng.standard_normal((12, 2, 4)) for _ in range(4))
    for causal in (False, True):
        ref = oracle.attention_backward(q, k, v, do, 0.45, causal)
        for w in (1, 2, 3, 4, 6):
            got = oracle.ring_attention_backward(q, k, v, do, 0.45, causal, w)
            for a, b in zip(got, ref):
                assert np.allclose(a, b, atol=1e-12, rtol=0)
    # planted mistakes, checked against the same definition
    def ring_bwd_variant(q, k, v, do, scale, causal, world, own_lse=False, no_skip=False, no_d=False):
        Q, K, V, dO = (np.asarray(x, dtype=np.float64) for x in (q, k, v, do))
        L, H, d = Q.shape
        S = L // world
        O, LSE = oracle.ring_attention_forward(Q, K, V, scale, causal, world)
        D = 0.0 * O.sum(axis=-1) if no_d else (dO * O).sum(axis=-1)
        dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
        for r in range(world):
            for s_ in range(world):
                if causal and s_ > r and not no_skip:
                    continue
                rows, cols = slice(r * S, (r + 1) * S), slice(s_ * S, (s_ + 1) * S)
                for h in range(H):
                    Sc = (Q[rows, h] @ K[cols, h].T) * scale
                    if causal and s_ == r:
                        Sc[np.triu_indices(S, k=1)] = -np.inf
                    lse = np.log(np.exp(Sc).sum(axis=1)) if own_lse else LSE[rows, h]
                    P = np.exp(Sc - lse[:, None])
                    dS = P * (dO[rows, h] @ V[cols, h].T - D[rows, h][:, None])
                    dQ[rows, h] += scale * (dS @ K[cols, h])
                    dK[cols, h] += scale * (dS.T @ Q[rows, h])
                    dV[cols, h] += P.T @ dO[rows, h]
        return dQ, dK, dV
    ref = oracle.attention_backward(q, k, v, do, 0.45, True)
    ok = lambda got: all(np.allclose(a, b, atol=1e-9, rtol=0) for a, b in zip(got, ref))
    assert ok(ring_bwd_variant(q, k, v, do, 0.45, True, 3))
    for kw in (dict(own_lse=True), dict(no_skip=True), dict(no_d=True)):
        assert not ok(ring_bwd_variant(q, k, v, do, 0.45, True, 3, **kw)), kw


# ----------------------------------------------------------------------------- load-balanced (zigzag) ring


def _zigzag_pins_pass(ring_fwd, ring_bwd, blocks):
    """Pins of the zigzag ring layout against the whole-sequence definition and the work balance."""
    rng = np.random.default_rng(77)
    H, d = 2, 4
    for w in (1, 2, 3, 4, 6):
        L = 2 * w * 3  # 3 tokens per chunk
        q, k, v, do = (rng.standard_normal((L, H, d)) for _ in range(4))
        for causal in (False, True):
            O, LSE = oracle.attention_forward(q, k, v, 0.6, causal)
            Oz, Lz = ring_fwd(q, k, v, 0.6, causal, w, "zigzag")
            if not (np.allclose(Oz, O, atol=1e-12) and np.allclose(Lz, LSE, atol=1e-12)):
                return False
            g = oracle.attention_backward(q, k, v, do, 0.6, causal)
            gz = ring_bwd(q, k, v, do, 0.6, causal, w, "zigzag")
            if not all(np.allclose(a, b, atol=1e-11) for a, b in zip(gz, g)):
                return False
        # every visible chunk pair is computed exactly once over the ring, and under the causal mask
        # every rank attends to the same number of (query, key) pairs
        C = 3
        work = []
        for causal in (False, True):
            seen = {}
            for r in range(w):
                pairs = 0
                for t in range(w):
                    s_ = (r - t) % w
                    for qi, ki, diag in blocks(r, t, w, causal, "zigzag"):
                        qc, kc = oracle.zigzag_chunks(r, w)[qi], oracle.zigzag_chunks(s_, w)[ki]
                        seen[(qc, kc)] = seen.get((qc, kc), 0) + 1
                        if diag != (causal and qc == kc):
                            return False
                        pairs += C * (C + 1) // 2 if diag else C * C
                work.append((causal, pairs))
            want = {(a, b) for a in range(2 * w) for b in range(2 * w) if not causal or b <= a}
            if set(seen) != want or any(n != 1 for n in seen.values()):
                return False
        causal_work = [p for c, p in work if c]
        if len(set(causal_work)) != 1:
            return False
    return True


def test_zigzag_ring_pins():
    assert _zigzag_pins_pass(oracle.ring_attention_forward, oracle.ring_attention_backward, oracle.ring_blocks)


def test_contiguous_ring_is_unbalanced_under_the_causal_mask():
    """The reason for the zigzag layout: with contiguous shards rank W-1 does W blocks, rank 0 one."""
    w = 4
    n = [len([1 for t in range(w) for _ in oracle.ring_blocks(r, t, w, True)]) for r in range(w)]
    assert n == [1, 2, 3, 4]
    z = [sum(2 if not diag else 1 for t in range(w) for (_, _, diag) in oracle.ring_blocks(r, t, w, True, "zigzag"))
         for r in range(w)]
    assert len(set(z)) == 1  # full blocks count 2 half-blocks, diagonal ones 1: equal for every rank


def test_zigzag_pins_catch_planted_mistakes():
    def blocks_variant(chunks, skip_side="greater", diag_rule=True):
        def blocks(rank, step, world, causal, layout="contiguous"):
            s_ = (rank - step) % world
            out = []
            for qi, qc in enumerate(chunks(rank, world)):
                for ki, kc in enumerate(chunks(s_, world)):
                    if causal and ((kc > qc) if skip_side == "greater" else (kc < qc)):
                        continue
                    out.append((qi, ki, causal and kc == qc if diag_rule else False))
            return out
        return blocks

    def ring_pair(chunks, **kw):
        blocks = blocks_variant(chunks, **kw)

        def parts(L, world):
            C = L // (2 * world)
            return [[(c * C, (c + 1) * C) for c in chunks(r, world)] for r in range(world)]

        def fwd(q, k, v, scale, causal, world, layout):
            Q, K, V = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
            L, H, d = Q.shape
            po = parts(L, world)
            O, LSE = np.zeros((L, H, d)), np.full((L, H), -np.inf)
            for r in range(world):
                acc = [[] for _ in po[r]]
                for t in range(world):
                    s_ = (r - t) % world
                    for qi, ki, diag in blocks(r, t, world, causal):
                        rows, cols = slice(*po[r][qi]), slice(*po[s_][ki])
                        acc[qi].append(oracle.attention_forward(Q[rows], K[cols], V[cols], scale, diag))
                for qi, (a, b) in enumerate(po[r]):
                    if acc[qi]:
                        O[a:b], LSE[a:b] = oracle.merge_attention_partials(acc[qi])
            return O, LSE

        def bwd(q, k, v, do, scale, causal, world, layout):
            return oracle.ring_attention_backward(q, k, v, do, scale, causal, world, layout)
        return fwd, bwd, blocks

    good = ring_pair(oracle.zigzag_chunks)
    assert _zigzag_pins_pass(*good)  # the restatement passes
    shifted = lambda r, w: (r, (2 * w - 2 - r) % (2 * w))  # the second chunk off by one
    for bad in (ring_pair(shifted), ring_pair(oracle.zigzag_chunks, skip_side="less"),
                ring_pair(oracle.zigzag_chunks, diag_rule=False)):
        assert not _zigzag_pins_pass(*bad)
