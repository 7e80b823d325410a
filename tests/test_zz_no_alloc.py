"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory.

Some users of this library run inside a host engine that owns all of the
GPU's memory and hands them only their input and output buffers, or must not
call cudaMalloc at all (it can synchronise the device and can fail under a
fixed memory budget).  fa_bwd_noalloc lets them run the backward with its
workspace in the library's own static device array instead of a buffer they
would have to allocate.  These tests call it through the C ABI and check that
it gives the same gradients as fa_bwd with a caller-provided workspace and,
within the gradient tolerance, as the fp64 oracle, on two calls in a row (the
array keeps the previous call's contents, so the second call shows that stale
scratch does no harm); and that, once the library is loaded, the calls change
neither the device's free memory nor PyTorch's allocations.  This file is
named to be collected last.
"""

import pytest
import torch

import workloads
from _gpu import GRAD_TOL, covered_rows, f64, oracle_backward, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    m = load_fa()
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for the gpu-marked tests")
    return m


def _ptr(t):
    return None if t is None else t.data_ptr()


@pytest.mark.parametrize("d,causal,dtype,seqlens", [
    (128, True, "bf16", None),
    (64, False, "fp16", None),
    (128, True, "bf16", [1, 300, 0, 129, 77]),
])
def test_noalloc_matches_workspace_backward_twice(fa, d, causal, dtype, seqlens):
    inp = workloads.random_inputs(3, d, dtype, seed=4242 + d, B=2, N=300, seqlens=seqlens, causal=causal)
    dev = torch.device("cuda")
    q, k, v, do = (t.to(dev) for t in (inp.q, inp.k, inp.v, inp.do))
    cu = None if inp.cu_seqlens is None else inp.cu_seqlens.to(dev)
    stream = torch.cuda.current_stream().cuda_stream
    B, H, N, T = inp.B, inp.H, inp.N, inp.T
    code = fa.dtype_code(q)
    o, lse = fa.attention_forward(q, k, v, causal=causal, scale=inp.scale, cu_seqlens=cu,
                                  max_seqlen=N if cu is not None else None, batch=B)
    # the existing entry point, with a workspace the caller allocated
    ws_bytes = fa.fa_bwd_workspace_bytes(T, H, d)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    ref = [torch.empty_like(q) for _ in range(3)]
    st = fa.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), *(_ptr(t) for t in ref), B, H, N, d,
                   inp.scale, int(causal), _ptr(cu), T, code, _ptr(ws), ws_bytes, stream)
    assert st == fa.FA_OK
    assert fa.fa_check_device_status(stream) == fa.FA_OK
    assert ws_bytes <= fa.FA_NOALLOC_SCRATCH_BYTES
    rows = covered_rows(inp)
    oracle_grads = oracle_backward(inp)
    outs = [[torch.full_like(q, float("nan")) for _ in range(3)] for _ in range(2)]
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    torch_before = torch.cuda.memory_allocated()
    for call in range(2):
        got = outs[call]
        st = fa.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), *(_ptr(t) for t in got),
                               B, H, N, d, inp.scale, int(causal), _ptr(cu), T, code, stream)
        assert st == fa.FA_OK, fa.fa_status_string(st)
        assert fa.fa_check_device_status(stream) == fa.FA_OK
    # nothing was allocated by the two calls (the library and its static array were loaded by the
    # first fa_bwd call above)
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.cuda.memory_allocated() == torch_before
    for call in range(2):
        for name, g, r, ro in zip(("dq", "dk", "dv"), outs[call], ref, oracle_grads):
            a = f64(g)[rows]
            e = rel_l2(a, f64(r)[rows])
            assert e <= GRAD_TOL, (call, name, "vs fa_bwd", e)
            e = rel_l2(a, ro[rows])
            assert e <= GRAD_TOL, (call, name, "vs oracle", e)


def test_noalloc_rejects_problems_beyond_its_scratch(fa):
    """A problem whose workspace exceeds FA_NOALLOC_SCRATCH_BYTES is refused before anything runs."""
    H, d = 16, 128
    T = fa.FA_NOALLOC_SCRATCH_BYTES // (H * d * 4) + 64  # the fp32 dQ accumulator alone is too large
    assert fa.fa_bwd_workspace_bytes(T, H, d) > fa.FA_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20  # never dereferenced: the size check comes first
    st = fa.fa_bwd_noalloc(*([fake] * 9), 1, H, T, d, 0.088, 1, None, T, fa.FA_BF16,
                           torch.cuda.current_stream().cuda_stream)
    assert st == fa.FA_ERR_UNSUPPORTED
