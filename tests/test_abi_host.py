"""Host-side checks of the C ABI: no GPU needed, no kernel launched.

The library must load, export every function ``include/fa.h`` declares, and
reject invalid arguments synchronously (before any CUDA call), so these run on
a machine without a GPU.
"""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(fa_[a-z0-9_]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def fa():
    from _lib import load_fa
    return load_fa()


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for n in ["fa_fwd", "fa_bwd", "fa_bwd_workspace_bytes", "fa_bwd_preprocess", "fa_bwd_main",
              "fa_bwd_postprocess", "fa_check_device_status", "fa_status_string", "fa_set_watchdog_ns",
              "fa_watchdog_selftest", "fa_version", "fa_bwd_noalloc", "fa_decode", "fa_decode_workspace_bytes",
              "fa_fwd_dropout", "fa_bwd_dropout", "fa_fwd_fp8", "fa_fwd_fp8_per_head", "fa_fwd_fp8_per_block",
              "fa_attn_merge",
              "fa_accumulate"]:
        assert n in names


def test_library_exports_every_declared_symbol(fa):
    lib = ctypes.CDLL(fa.LIB_PATH)
    for n in _declared_functions():
        assert hasattr(lib, n), f"{n} declared in fa.h but not exported"


def test_status_strings(fa):
    assert fa.fa_status_string(0) == "FA_OK"
    assert fa.fa_status_string(4) == "FA_ERR_TIMEOUT"
    assert fa.fa_status_string(99) == "FA_UNKNOWN_STATUS"
    assert "sm_100a" in fa.fa_version()


def test_workspace_bytes(fa):
    # fp32 dQ accumulator [T,H,d] + fp32 D [T,H], each rounded up to 256 bytes
    def up(x):
        return (x + 255) // 256 * 256
    assert fa.fa_bwd_workspace_bytes(32768 * 1, 16, 128) == up(32768 * 16 * 128 * 4) + up(32768 * 16 * 4)
    assert fa.fa_bwd_workspace_bytes(3, 1, 64) == up(3 * 64 * 4) + up(3 * 4)
    assert fa.fa_bwd_workspace_bytes(0, 16, 128) == 0
    assert fa.fa_bwd_workspace_bytes(16, 16, 96) == 0


GOOD = dict(B=2, H=4, N=256, d=64, scale=0.125, causal=0, cu=None, T=512, dtype=0)
P16 = 1 << 20  # a fake, 16-byte aligned "device" address: never dereferenced (validation fails first)


def _fwd(fa, **kw):
    a = dict(GOOD)
    a.update(kw)
    ptrs = a.pop("ptrs", [P16] * 5)
    return fa.fa_fwd(*ptrs, a["B"], a["H"], a["N"], a["d"], a["scale"], a["causal"], a["cu"], a["T"], a["dtype"], None)


@pytest.mark.parametrize("bad", [
    dict(d=96), dict(d=0), dict(B=0), dict(H=0), dict(N=0), dict(T=0), dict(T=511),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(scale=0.0), dict(scale=-1.0),
    dict(causal=2), dict(causal=-1), dict(dtype=2),
    dict(ptrs=[0, P16, P16, P16, P16]), dict(ptrs=[P16, P16, P16, P16, 0]),
    dict(ptrs=[P16 + 8, P16, P16, P16, P16]), dict(ptrs=[P16, P16, P16 + 2, P16, P16]),
    dict(ptrs=[P16, P16, P16, P16, P16 + 2]), dict(cu=P16 + 2),
])
def test_forward_rejects_invalid_arguments(fa, bad):
    assert _fwd(fa, **bad) == fa.FA_ERR_INVALID_ARG


def test_backward_rejects_invalid_arguments(fa):
    ws = fa.fa_bwd_workspace_bytes(512, 4, 64)
    args = [P16] * 9 + [2, 4, 256, 64, 0.125, 0, None, 512, 0, P16, ws, None]
    assert fa.fa_bwd(*args[:19], ws - 1, None) == fa.FA_ERR_INVALID_ARG          # workspace too small
    bad_ws = list(args)
    bad_ws[18] = P16 + 16                                                        # workspace not 256-byte aligned
    assert fa.fa_bwd(*bad_ws) == fa.FA_ERR_INVALID_ARG
    bad_d = list(args)
    bad_d[12] = 80
    assert fa.fa_bwd(*bad_d) == fa.FA_ERR_INVALID_ARG
    null_dq = list(args)
    null_dq[6] = 0
    assert fa.fa_bwd(*null_dq) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_preprocess(P16, P16, 2, 4, 256, 64, None, 512, 0, P16, ws - 256, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_postprocess(P16, 2, 4, 256, 64, float("nan"), None, 512, 0, P16, ws, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_main(P16, P16, P16, P16, P16, P16, P16, 2, 4, 256, 64, 0.125, 3, None, 512, 0, P16, ws,
                          None) == fa.FA_ERR_INVALID_ARG


def test_dropout_rejects_invalid_probability(fa):
    args = [P16] * 5 + [2, 4, 256, 64, 0.125, 0, None, 512, 0]
    for p in (-0.1, 1.0, 1.5, float("nan")):
        assert fa.fa_fwd_dropout(*args, p, 1, 0, None) == fa.FA_ERR_INVALID_ARG
    ws = fa.fa_bwd_workspace_bytes(512, 4, 64)
    bargs = [P16] * 9 + [2, 4, 256, 64, 0.125, 0, None, 512, 0]
    assert fa.fa_bwd_dropout(*bargs, 1.0, 1, 0, P16, ws, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_bwd_dropout(*bargs, 0.1, 1, 0, P16, ws - 1, None) == fa.FA_ERR_INVALID_ARG


def test_fp8_rejects_invalid_arguments(fa):
    args = [P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 512]
    for ds in (0.0, -1.0, float("nan"), float("inf")):
        assert fa.fa_fwd_fp8(*args, ds, 1.0, 1.0, None) == fa.FA_ERR_INVALID_ARG
        assert fa.fa_fwd_fp8(*args, 1.0, ds, 1.0, None) == fa.FA_ERR_INVALID_ARG
        assert fa.fa_fwd_fp8(*args, 1.0, 1.0, ds, None) == fa.FA_ERR_INVALID_ARG
    # the folded softmax scale must stay finite
    assert fa.fa_fwd_fp8(*args, 1e30, 1e30, 1.0, None) == fa.FA_ERR_INVALID_ARG
    # e4m3 inputs are built for d = 128 only
    assert fa.fa_fwd_fp8(*([P16] * 5 + [2, 4, 256, 64, 0.125, 0, None, 512]), 1.0, 1.0, 1.0, None) == \
        fa.FA_ERR_UNSUPPORTED
    # misaligned pointer, bad causal flag, token count mismatch
    assert fa.fa_fwd_fp8(*([P16 + 8] + [P16] * 4 + [2, 4, 256, 128, 0.125, 0, None, 512]), 1.0, 1.0, 1.0, None) == \
        fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8(*([P16] * 5 + [2, 4, 256, 128, 0.125, 2, None, 512]), 1.0, 1.0, 1.0, None) == \
        fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8(*([P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 511]), 1.0, 1.0, 1.0, None) == \
        fa.FA_ERR_INVALID_ARG


def test_fp8_per_head_rejects_invalid_arguments(fa):
    base = [P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 512]
    for i, bad in [(0, None), (1, P16 + 2), (2, None)]:  # q, k, v descale arrays: null or misaligned
        ds = [P16, P16, P16]
        ds[i] = bad
        assert fa.fa_fwd_fp8_per_head(*base, *ds, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8_per_head(*([P16] * 5 + [2, 4, 256, 64, 0.125, 0, None, 512]), P16, P16, P16, None) == \
        fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_fp8_per_head(*([P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 511]), P16, P16, P16, None) == \
        fa.FA_ERR_INVALID_ARG


def test_fp8_per_block_rejects_invalid_arguments(fa):
    base = [P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 512]
    for i, bad in [(0, None), (1, P16 + 2), (2, None)]:  # q, k, v descale arrays: null or misaligned
        ds = [P16, P16, P16]
        ds[i] = bad
        assert fa.fa_fwd_fp8_per_block(*base, *ds, 4, None) == fa.FA_ERR_INVALID_ARG
    # a dense batch of 2 × 256 tokens has 2·2 blocks: 3 is too few, 0 is never valid
    assert fa.fa_fwd_fp8_per_block(*base, P16, P16, P16, 3, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8_per_block(*base, P16, P16, P16, 0, None) == fa.FA_ERR_INVALID_ARG
    assert fa.fa_fwd_fp8_per_block(*([P16] * 5 + [2, 4, 256, 64, 0.125, 0, None, 512]), P16, P16, P16, 4, None) == \
        fa.FA_ERR_UNSUPPORTED
    assert fa.fa_fwd_fp8_per_block(*([P16] * 5 + [2, 4, 256, 128, 0.125, 0, None, 511]), P16, P16, P16, 4, None) == \
        fa.FA_ERR_INVALID_ARG


def test_merge_rejects_invalid_arguments(fa):
    ok = [P16, P16, P16, P16, None, 64, 4, 128, 0, 0, None]
    for i, bad in [(0, P16 + 4), (2, P16 + 8), (1, P16 + 2), (3, 0), (4, P16 + 8)]:
        args = list(ok)
        args[i] = bad
        assert fa.fa_attn_merge(*args) == fa.FA_ERR_INVALID_ARG, i
    for i, bad in [(5, 0), (6, 0), (7, 96), (8, 7), (9, 2)]:
        args = list(ok)
        args[i] = bad
        assert fa.fa_attn_merge(*args) == fa.FA_ERR_INVALID_ARG, i


def test_accumulate_rejects_invalid_arguments(fa):
    for args in ([P16 + 4, P16, None, 4096, 0, 0], [P16, P16 + 8, None, 4096, 0, 0], [P16, None, P16 + 2, 4096, 0, 0],
                 [P16, P16, None, 4095, 0, 0], [P16, P16, None, 0, 0, 0], [P16, P16, None, 4096, 5, 0],
                 [P16, P16, None, 4096, 0, 3]):
        assert fa.fa_accumulate(*args, None) == fa.FA_ERR_INVALID_ARG, args


def test_decode_workspace_bytes(fa):
    # per (sequence, head, 512-key chunk): d fp32 partial outputs + (m, ℓ), each part rounded up to 256 bytes
    def up(x):
        return (x + 255) // 256 * 256
    slots = 16 * 16 * 16  # B = 16, H = 16, 8192 keys → 16 chunks
    assert fa.fa_decode_workspace_bytes(16, 16, 8192, 128) == up(slots * 128 * 4) + up(slots * 2 * 4)
    assert fa.fa_decode_workspace_bytes(1, 1, 513, 64) == up(2 * 64 * 4) + up(2 * 2 * 4)
    assert fa.fa_decode_workspace_bytes(0, 16, 8192, 128) == 0
    assert fa.fa_decode_workspace_bytes(1, 1, 64, 96) == 0


def test_decode_rejects_invalid_arguments(fa):
    ws = fa.fa_decode_workspace_bytes(2, 4, 256, 64)
    good = dict(q=P16, k=P16, v=P16, o=P16, lse=P16, B=2, H=4, Nk=256, d=64, scale=0.125, cu_seqlens_k=None,
                total_keys=512, dtype=0, workspace=P16, workspace_bytes=ws, stream=None)
    for bad in [dict(d=96), dict(B=0), dict(Nk=0), dict(total_keys=511), dict(scale=float("nan")), dict(scale=0.0),
                dict(dtype=3), dict(q=0), dict(k=P16 + 8), dict(lse=P16 + 2), dict(workspace=P16 + 16),
                dict(workspace_bytes=ws - 1), dict(cu_seqlens_k=P16 + 2)]:
        a = dict(good)
        a.update(bad)
        assert fa.fa_decode(**a) == fa.FA_ERR_INVALID_ARG, bad
    a = dict(good)
    a.update(B=70000, total_keys=70000 * 256, workspace_bytes=fa.fa_decode_workspace_bytes(70000, 4, 256, 64))
    assert fa.fa_decode(**a) == fa.FA_ERR_UNSUPPORTED


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    """The binding has no fallback: without the shared library the import raises."""
    import importlib.util
    import shutil
    pkg = os.path.join(ROOT, "exact_io_aware_90_b200")
    dst = tmp_path / "exact_io_aware_90_b200"
    os.makedirs(dst)
    shutil.copy(os.path.join(pkg, "__init__.py"), dst / "__init__.py")  # no .so beside it
    spec = importlib.util.spec_from_file_location("fa_copy_without_lib", dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="missing"):
        spec.loader.exec_module(mod)
