"""GPU tests of the device-side check of inconsistent cu_seqlens (the varlen interface).

The host cannot read cu_seqlens without a device-to-host copy, so each kernel
checks every sequence it works on: a sequence whose offsets decrease, whose
end lies past the token count T, or whose length exceeds N (the maximum the
call declares) is skipped, and FA_ERR_INVALID_ARG is recorded in the device
status word that fa_check_device_status returns.  These tests pass such
offsets to the forward, the backward and decode through the C ABI and check
that the status is recorded, that rows no valid sequence covers keep the
caller's values, that nothing faults, and that a valid call right after
works.  Each kernel skips the bad sequence before touching memory, so no
case reads or writes outside the caller's buffers.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu

T, H, N = 512, 2, 256
# offsets (B + 1 entries) and the rows no valid sequence covers
CASES = {
    "decreasing": ([0, 200, 100, 300], range(300, T)),      # sequence 1 has a negative length
    "past_T": ([0, 100, T + 64], range(100, T)),            # sequence 1 ends past T
    "longer_than_N": ([0, N + 1, N + 11], list(range(0, N + 1)) + list(range(N + 11, T))),  # sequence 0 > N
}
SENTINEL = 7.0


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    m.fa_set_watchdog_ns(1_000_000_000)  # a wait that never completes returns FA_ERR_TIMEOUT, not a hang
    return m


def _inputs(d, seed):
    g = torch.Generator().manual_seed(seed)
    dev = torch.device("cuda")
    q, k, v, do = (torch.randn(T, H, d, generator=g).to(torch.bfloat16).to(dev) for _ in range(4))
    return q, k, v, do


def _status(fa):
    return fa.fa_check_device_status(torch.cuda.current_stream().cuda_stream)


def _valid_call_works(fa, d):
    q, k, v, _ = _inputs(d, 5)
    cu = torch.tensor([0, 100, T], dtype=torch.int32, device="cuda")
    fa.attention_forward(q, k, v, causal=True, cu_seqlens=cu, max_seqlen=T, batch=2)
    assert _status(fa) == fa.FA_OK


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("d", [64, 128])
def test_forward_records_bad_offsets(fa, case, d):
    offsets, uncovered = CASES[case]
    q, k, v, _ = _inputs(d, 11)
    cu = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    o = torch.full_like(q, SENTINEL)
    lse = torch.full((T, H), SENTINEL, dtype=torch.float32, device="cuda")
    assert _status(fa) == fa.FA_OK
    fa.attention_forward(q, k, v, causal=True, cu_seqlens=cu, max_seqlen=N, batch=len(offsets) - 1, out=o, lse=lse)
    assert _status(fa) == fa.FA_ERR_INVALID_ARG
    rows = torch.tensor(list(uncovered), device="cuda")
    assert torch.all(o[rows].float() == SENTINEL) and torch.all(lse[rows] == SENTINEL)
    _valid_call_works(fa, d)


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("d", [64, 128])
def test_backward_records_bad_offsets(fa, case, d):
    offsets, uncovered = CASES[case]
    q, k, v, do = _inputs(d, 12)
    o = torch.randn_like(q.float()).to(torch.bfloat16)
    lse = torch.zeros((T, H), dtype=torch.float32, device="cuda")
    cu = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    dq, dk, dv = (torch.full_like(q, SENTINEL) for _ in range(3))
    assert _status(fa) == fa.FA_OK
    fa.attention_backward(q, k, v, o, lse, do, causal=True, cu_seqlens=cu, max_seqlen=N, batch=len(offsets) - 1,
                          dq=dq, dk=dk, dv=dv)
    assert _status(fa) == fa.FA_ERR_INVALID_ARG
    rows = torch.tensor(list(uncovered), device="cuda")
    # dK and dV rows of a skipped sequence keep the caller's values (dQ is written from the zeroed
    # accumulator for every row up to min(T, cu_seqlens[B]))
    assert torch.all(dk[rows].float() == SENTINEL) and torch.all(dv[rows].float() == SENTINEL)
    assert torch.all(torch.isfinite(dq.float()))
    _valid_call_works(fa, d)


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("d", [64, 128])
def test_decode_records_bad_offsets(fa, case, d):
    offsets, _ = CASES[case]
    B = len(offsets) - 1
    _, k, v, _ = _inputs(d, 13)
    q = torch.randn(B, H, d).to(torch.bfloat16).cuda()
    cu = torch.tensor(offsets, dtype=torch.int32, device="cuda")
    o = torch.full_like(q, SENTINEL)
    lse = torch.full((B, H), SENTINEL, dtype=torch.float32, device="cuda")
    assert _status(fa) == fa.FA_OK
    fa.attention_decode(q, k, v, cu_seqlens_k=cu, max_seqlen_k=N, out=o, lse=lse)
    assert _status(fa) == fa.FA_ERR_INVALID_ARG
    bad = [b for b in range(B) if not (0 <= offsets[b] <= offsets[b + 1] <= T and offsets[b + 1] - offsets[b] <= N)]
    assert bad
    for b in bad:  # the skipped sequence's output keeps the caller's values
        assert torch.all(o[b].float() == SENTINEL) and torch.all(lse[b] == SENTINEL)
    _valid_call_works(fa, d)
