"""GPU parity of decode (one query per sequence, split-KV) against the fp64 oracle, through the C ABI.

Key counts straddle the 512-key chunks (1, 511, 512, 513, several chunks), packed batches hold empty
sequences, and the full-size decode workloads are compared on every (sequence, head).
"""

import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from _gpu import LSE_TOL, O_TOL, f64, max_abs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    m.fa_set_watchdog_ns(2_000_000_000)
    return m


def _run(fa, inp):
    dev = torch.device("cuda")
    q, k, v = inp.q.to(dev), inp.k.to(dev), inp.v.to(dev)
    cu = None if inp.cu_seqlens_k is None else inp.cu_seqlens_k.to(dev)
    o, lse = fa.attention_decode(q, k, v, scale=inp.scale, cu_seqlens_k=cu,
                                 max_seqlen_k=inp.Nk if cu is not None else None)
    st = fa.fa_check_device_status(torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_OK, fa.fa_status_string(st)
    return o, lse


def _check(fa, inp):
    o, lse = _run(fa, inp)
    cu = None if inp.cu_seqlens_k is None else inp.cu_seqlens_k.numpy()
    O_ref, L_ref = oracle.decode_forward(inp.q, inp.k, inp.v, inp.scale, cu_seqlens_k=cu, B=inp.B,
                                         Nk=inp.Nk if cu is None else None)
    go, gl = f64(o), f64(lse)
    assert max_abs(go, O_ref) <= O_TOL, max_abs(go, O_ref)
    fin = np.isfinite(L_ref)
    assert np.array_equal(np.isfinite(gl), fin)
    assert np.all(np.abs(gl[fin] - L_ref[fin]) <= LSE_TOL), np.abs(gl[fin] - L_ref[fin]).max()
    assert np.all(go[~fin] == 0.0)
    return go, gl


@pytest.mark.parametrize("Nk", [1, 7, 511, 512, 513, 1500, 4097])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_decode_shapes(fa, Nk, d, dtype):
    inp = workloads.decode_inputs(3, d, dtype, seed=Nk + d, B=2, Nk=Nk, scale=2.0 / math.sqrt(d))
    _check(fa, inp)


@pytest.mark.parametrize("d", [64, 128])
def test_decode_varlen_with_empty_sequences(fa, d):
    inp = workloads.decode_inputs(4, d, "bf16", seed=77, seqlens=[0, 1, 512, 0, 513, 2049, 37, 0])
    go, gl = _check(fa, inp)
    for b in (0, 3, 7):  # no key: O = 0, LSE = -inf
        assert np.all(go[b] == 0.0) and np.all(np.isneginf(gl[b]))


def test_decode_large_scores_are_stable(fa):
    inp = workloads.decode_inputs(2, 128, "bf16", seed=5, B=2, Nk=3000, scale=8.0 / math.sqrt(128))
    _check(fa, inp)


def test_decode_hand_example(fa):
    """The narration's example as one decode step: exponentiated scores [1, 2, 4, 3], values
    [10, 20, 30, 40] give 29 (fp16 holds 29 to 1/64)."""
    inp = workloads.hand_example_inputs("fp16")
    dev = torch.device("cuda")
    o, lse = fa.attention_decode(inp.q[:1].to(dev), inp.k.to(dev), inp.v.to(dev), scale=inp.scale)
    assert abs(float(o[0, 0, 0]) - 29.0) <= 0.03
    assert abs(float(lse[0, 0]) - math.log(10.0)) <= 5e-3


@pytest.mark.parametrize("name", ["decode_b16_kv8k", "decode_varlen"])
def test_decode_workloads(fa, name):
    _check(fa, workloads.make_decode_workload(name))


def test_decode_repeatable(fa):
    inp = workloads.decode_inputs(4, 128, "bf16", seed=9, B=3, Nk=5000)
    o1, l1 = _run(fa, inp)
    o1, l1 = o1.clone(), l1.clone()
    o2, l2 = _run(fa, inp)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_argument_checks(fa):
    dev = torch.device("cuda")
    q = torch.zeros(2, 2, 128, dtype=torch.bfloat16, device=dev)
    k = torch.zeros(8, 2, 128, dtype=torch.bfloat16, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty(2, 2, dtype=torch.float32, device=dev)
    ws = torch.empty(fa.fa_decode_workspace_bytes(2, 2, 4, 128), dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    args = lambda **kw: dict(dict(q=q.data_ptr(), k=k.data_ptr(), v=k.data_ptr(), o=o.data_ptr(),
                                  lse=lse.data_ptr(), B=2, H=2, Nk=4, d=128, scale=0.1, cu_seqlens_k=None,
                                  total_keys=8, dtype=fa.FA_BF16, workspace=ws.data_ptr(),
                                  workspace_bytes=ws.numel(), stream=s), **kw)
    assert fa.fa_decode(**args()) == fa.FA_OK
    assert fa.fa_decode(**args(d=96)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_decode(**args(total_keys=9)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_decode(**args(workspace_bytes=ws.numel() - 1)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_decode(**args(scale=float("nan"))) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_decode(**args(q=q.data_ptr() + 2)) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_check_device_status(s) == fa.FA_OK
