"""Seeded input generator: pinned to its published definitions (SplitMix64, Box-Muller, RNE)."""
import math

import numpy as np
import pytest

import seeded_inputs as si


def _mix(z):
    M = (1 << 64) - 1
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    return z ^ (z >> 31)


def test_splitmix64_reference_outputs():
    # Published SplitMix64 with state 0: first outputs of the generator.
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1
    assert _mix(G & M) == 0xE220A8397B1DCDAF
    assert _mix((2 * G) & M) == 0x6E789E6AA1B965F4
    # the library's draws are outputs of a stream whose state is output `stream` of a seed generator
    for seed, stream, ctr in ((0, 0, 0), (7, 3, 12345), (2**63 + 5, 4, 2**40)):
        state = _mix((seed + (stream + 1) * G) & M)
        assert si.draw_u64(seed, stream, ctr) == _mix((state + (ctr + 1) * G) & M)


def test_box_muller_against_libm():
    G = 0x9E3779B97F4A7C15
    M = (1 << 64) - 1
    seed, stream = 0, 1
    vals = si.fill_host((64,), seed, stream, bf16=False)
    state = _mix((seed + (stream + 1) * G) & M)
    for i in range(64):
        z = _mix((state + (i // 2 + 1) * G) & M)
        u1 = ((z >> 40) + 1) / 2**24
        u2 = ((z >> 16) & 0xFFFFFF) / 2**24
        r = math.sqrt(-2 * math.log(u1))
        x = r * (math.sin if i & 1 else math.cos)(2 * math.pi * u2)
        assert abs(float(vals[i]) - x) <= 1e-6 * max(1.0, abs(x))
        assert vals[i] == np.float32(x) or abs(float(vals[i]) - x) < 2e-7 * max(1, abs(x))


def test_moments_and_uniform_range():
    x = si.fill_host((1 << 20,), 3, 0, bf16=False)
    assert abs(x.mean()) < 0.005 and abs(x.std() - 1) < 0.005
    # tail mass beyond 3 sigma: 0.27 %
    assert abs((np.abs(x) > 3).mean() - 0.0027) < 0.0006
    y = si.fill_host((1 << 20,), 3, 0, a=1.0, b=2.5, bf16=False)
    np.testing.assert_allclose(y, 1.0 + 2.5 * x.astype(np.float64), rtol=1e-6, atol=1e-6)
    u = si.fill_host((1 << 20,), 3, 2, kind=si.UNIFORM, a=-1, b=1, bf16=False)
    assert u.min() >= -1 and u.max() < 1 and abs(u.mean()) < 0.005


def test_bf16_rounding_is_rne():
    x = si.fill_host((4096,), 5, 0, bf16=False)
    b = si.fill_host((4096,), 5, 0, bf16=True)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    expect = ((bits + 0x7FFF + lsb) >> 16).astype(np.uint16)
    np.testing.assert_array_equal(b, expect)
    # widening is exact and within half a bf16 ulp of the float32 value
    w = si.bf16_bits_to_f32(b)
    assert (np.abs(w - x) <= np.abs(x) * 2.0**-8).all()


def test_counter_offsets_and_threads():
    full = si.fill_host((10000,), 9, 2, threads=4)
    part = si.fill_host((3000,), 9, 2, start=5001, threads=1)
    np.testing.assert_array_equal(full[5001:8001], part)


def test_lengths_and_rows():
    lens = si.kv_lengths(64, 1024, 16384)
    assert lens.min() >= 1024 and lens.max() <= 16384
    np.testing.assert_array_equal(lens, si.kv_lengths(64, 1024, 16384))
    rows = si.sample_rows(8192, 256, salt=3)
    assert len(rows) == 256 and len(set(rows.tolist())) == 256
    assert rows[0] == 0 and rows[-1] == 8191 and (np.diff(rows) > 0).all()
    assert (si.sample_rows(8192, 256, salt=4) != rows).any()


@pytest.mark.gpu
def test_device_generator_matches_host_bits(cuda_device):
    import torch
    n = 3 * 65536 + 17
    for kind, a, b in ((si.NORMAL, 0.0, 1.0), (si.NORMAL, 0.0, 2.5), (si.UNIFORM, -1.0, 1.0)):
        t = torch.empty(n, dtype=torch.bfloat16, device=cuda_device)
        si.fill_device(t, 0, 1, kind, a, b, start=12)
        host = si.fill_host((n,), 0, 1, kind, a, b, bf16=True, start=12)
        np.testing.assert_array_equal(t.view(torch.int16).cpu().numpy().view(np.uint16), host)
        f = torch.empty(n, dtype=torch.float32, device=cuda_device)
        si.fill_device(f, 0, 1, kind, a, b, start=12)
        np.testing.assert_array_equal(f.cpu().numpy(), si.fill_host((n,), 0, 1, kind, a, b, bf16=False, start=12))


@pytest.mark.gpu
def test_device_cache_fill(cuda_device):
    import torch
    B, H, n_cap, d = 3, 2, 40, 16
    lens = np.array([1, 40, 17], np.int32)
    t = torch.empty((B, H, n_cap, d), dtype=torch.bfloat16, device=cuda_device)
    si.fill_device_cache(t, torch.from_numpy(lens).to(cuda_device), 0, 1)
    got = t.view(torch.int16).cpu().numpy().view(np.uint16)
    full = si.fill_host((B, H, n_cap, d), 0, 1)
    for b in range(B):
        np.testing.assert_array_equal(got[b, :, :lens[b]], full[b, :, :lens[b]])
        assert (got[b, :, lens[b]:] == 0x7FC0).all()
