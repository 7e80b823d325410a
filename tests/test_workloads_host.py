"""Host checks of the seeded input generators (no GPU): the e4m3 quantisation both the kernels and the
oracle consume, and the determinism of every generator the tests and the benchmark use."""

import math

import numpy as np
import torch

import workloads


def test_e4m3_per_tensor_inputs():
    inp = workloads.random_inputs(2, 128, "e4m3", seed=5, B=2, N=300, causal=True, backward=False)
    for name, t in (("q", inp.q), ("k", inp.k), ("v", inp.v)):
        ds = inp.extra["descale"][name]
        assert t.dtype == torch.float8_e4m3fn
        assert ds == float(np.float32(ds)) and ds > 0                 # an fp32 value, as the C ABI receives it
        assert float(t.float().abs().max()) == workloads.E4M3_MAX   # amax maps to 448
    # the same seed gives the same bytes; another seed does not
    again = workloads.random_inputs(2, 128, "e4m3", seed=5, B=2, N=300, causal=True, backward=False)
    assert torch.equal(inp.q.view(torch.uint8), again.q.view(torch.uint8))
    other = workloads.random_inputs(2, 128, "e4m3", seed=6, B=2, N=300, causal=True, backward=False)
    assert not torch.equal(inp.q.view(torch.uint8), other.q.view(torch.uint8))


def test_e4m3_per_head_quantisation():
    """Each (sequence, head) is divided by its own amax/448: its largest stored magnitude is 448, and
    stored × descale reproduces the fp32 source within e4m3's rounding (relative 2⁻⁴, or half the
    smallest subnormal step 2⁻⁹·descale near zero)."""
    g = torch.Generator().manual_seed(3)
    segs = [(0, 100), (100, 0), (100, 257)]
    x = torch.randn(357, 3, 128, generator=g) * torch.tensor([1.0, 8.0, 0.125])[None, :, None]
    q8, ds = workloads.quantize_e4m3_per_head(x, segs)
    assert ds.shape == (3, 3) and ds.dtype == np.float32
    assert np.all(ds[1] == 1.0)                                       # the empty sequence keeps descale 1
    for b, (s0, L) in enumerate(segs):
        if L == 0:
            continue
        stored = q8[s0:s0 + L].float()
        assert torch.all(stored.abs().amax(dim=(0, 2)) == workloads.E4M3_MAX)
    real = workloads.real_values(q8, ds, segs)
    src = x.double().numpy()
    dsrow = np.concatenate([np.repeat(ds[b][None, :], L, axis=0) for b, (s0, L) in enumerate(segs)])[:, :, None]
    bound = 2.0 ** -4 * np.abs(src) + 2.0 ** -10 * dsrow
    assert np.all(np.abs(real - src) <= bound * (1 + 1e-6))
    # per head, the descales differ by the magnitudes the heads were drawn at
    assert math.isclose(float(ds[0, 1] / ds[0, 0]), 8.0, rel_tol=0.5)


def test_e4m3_quantisers_zero_heads_and_gaps():
    """An all-zero (sequence, head) keeps descale 1 and stores exact zeros (descale 0 would make NaN
    codes and break the kernels' 'finite and > 0' contract); tokens outside every segment are 0."""
    x = torch.randn(40, 2, 128, generator=torch.Generator().manual_seed(9))
    x[0:10, 1] = 0.0                                                   # head 1 of sequence 0 is all zero
    segs = [(0, 10), (10, 20)]                                         # tokens 30..39 belong to no segment
    q8, ds = workloads.quantize_e4m3_per_head(x, segs)
    assert ds[0, 1] == 1.0 and np.all(np.isfinite(ds)) and np.all(ds > 0)
    stored = q8.float()
    assert torch.all(torch.isfinite(stored))
    assert torch.all(stored[0:10, 1] == 0) and torch.all(stored[30:] == 0)


def test_generators_are_deterministic():
    for name in ("tiny_d64", "mha_n4k_d64"):
        a, b = workloads.make_workload(name), workloads.make_workload(name)
        assert torch.equal(a.q, b.q) and torch.equal(a.v, b.v)
    lens = workloads.varlen_lengths(32, 128, 4096, 1004)
    assert lens == workloads.varlen_lengths(32, 128, 4096, 1004) and min(lens) >= 128 and max(lens) <= 4096
    cu = workloads.cu_from_lengths(lens)
    assert cu.dtype == torch.int32 and int(cu[0]) == 0 and int(cu[-1]) == sum(lens)


def test_e4m3_per_block_quantisation():
    """Per-block descales: the blocks of each sequence are its tokens [128i, 128i + 128) (the last one
    ragged), numbered sequence after sequence; each (block, head) has its largest stored magnitude at
    448, and stored × descale reproduces the source within e4m3's rounding."""
    assert workloads.block_segments([(0, 200), (200, 0), (200, 513), (713, 64)]) == \
        [(0, 128), (128, 72), (200, 128), (328, 128), (456, 128), (584, 128), (712, 1), (713, 64)]
    g = torch.Generator().manual_seed(4)
    segs = [(0, 200), (200, 0), (200, 300)]
    x = torch.randn(500, 2, 128, generator=g)
    x[128:200] *= 16.0                                                # the second block of sequence 0
    q8, ds = workloads.quantize_e4m3_per_block(x, segs)
    blocks = workloads.block_segments(segs)
    assert ds.shape == (len(blocks), 2) == (5, 2)
    for n, (s0, L) in enumerate(blocks):
        assert torch.all(q8[s0:s0 + L].float().abs().amax(dim=(0, 2)) == workloads.E4M3_MAX)
    assert math.isclose(float(ds[1, 0] / ds[0, 0]), 16.0, rel_tol=0.5)
    real = workloads.real_values(q8, ds, blocks)
    dsrow = np.concatenate([np.repeat(ds[n][None, :], L, axis=0) for n, (s0, L) in enumerate(blocks)])[:, :, None]
    src = x.double().numpy()
    assert np.all(np.abs(real - src) <= (2.0 ** -4 * np.abs(src) + 2.0 ** -10 * dsrow) * (1 + 1e-6))
