"""sdpa_decode_noalloc: decode for callers that are not allowed to allocate device memory.

Some callers -- a plug-in whose host application owns every device allocation,
or code under a fixed memory budget where only a framework's allocator may
allocate -- cannot call cudaMalloc or keep a workspace buffer.  For them the
library offers sdpa_decode_noalloc, which keeps its split partials in one fixed
library-owned device array instead of a caller workspace.  These tests call it
through the C ABI and check it against sdpa_decode (caller-provided workspace)
on the same inputs, on consecutive calls that reuse the shared array, and, on
the full decode workload (whose partials at sdpa_decode's split length do not
fit the array, so the call lengthens its splits), against the CPU oracle.
"""
import ctypes
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs import workloads as W

pytestmark = pytest.mark.gpu

BF16_ATOL, BF16_RTOL, LSE_TOL = 1e-2, 1e-2, 1e-3


@pytest.fixture(scope="module")
def lib(cuda_device):
    import memory_optimal_sdpa_b200 as m
    return m.lib


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _decode_both(lib, dev, B, H, cap, d, lens, seed):
    import torch
    q = si.fill_host((B, H, d), seed, 0)
    k = si.fill_host((B, H, cap, d), seed, 1)
    v = si.fill_host((B, H, cap, d), seed, 2)
    for b in range(B):  # rows past the length are never read: make any read visible
        k[b, :, lens[b]:] = 0x7FC0
        v[b, :, lens[b]:] = 0x7FC0
    tq, tk, tv = (W.to_torch(x, dev) for x in (q, k, v))
    tl = torch.from_numpy(np.asarray(lens, np.int32)).to(dev)
    scale = float(np.float32(1 / math.sqrt(d)))
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # existing entry point, workspace from the caller
    o_ref = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)
    l_ref = torch.empty((B, H), dtype=torch.float32, device=dev)
    need = lib.sdpa_decode_workspace_size(B, H, cap, d)
    ws = torch.empty(need, dtype=torch.uint8, device=dev)
    assert lib.sdpa_decode(_p(tq), _p(tk), _p(tv), _p(tl), _p(o_ref), _p(l_ref), B, H, cap, d, d, scale, _p(ws),
                           need, st) == 0
    # allocation-free entry point
    o = torch.full((B, H, d), float("nan"), dtype=torch.bfloat16, device=dev)
    l = torch.full((B, H), float("nan"), dtype=torch.float32, device=dev)
    assert lib.sdpa_decode_noalloc(_p(tq), _p(tk), _p(tv), _p(tl), _p(o), _p(l), B, H, cap, d, d, scale, st) == 0
    assert lib.sdpa_get_last_device_error(st) == 0
    O, O_ref = o.float().cpu().numpy(), o_ref.float().cpu().numpy()
    assert np.isfinite(O).all()
    assert (np.abs(O - O_ref) <= BF16_ATOL + BF16_RTOL * np.abs(O_ref)).all(), np.abs(O - O_ref).max()
    assert np.abs(l.cpu().numpy() - l_ref.cpu().numpy()).max() <= LSE_TOL


def test_noalloc_matches_workspace_decode_on_consecutive_calls(lib, cuda_device):
    g = np.random.default_rng(1)
    # first call: 64 (batch, head) pairs, d = 128, a cache long enough to need several splits
    lens1 = g.integers(1, 4097, size=8).astype(np.int32)
    lens1[0], lens1[1] = 1, 4096
    _decode_both(lib, cuda_device, 8, 8, 4096, 128, lens1, seed=21)
    # second call reuses the shared array with another shape and head dim
    lens2 = g.integers(1, 2001, size=4).astype(np.int32)
    _decode_both(lib, cuda_device, 4, 6, 2000, 64, lens2, seed=22)


def test_noalloc_rejects_sizes_beyond_its_scratch(lib, cuda_device):
    P = 0x10000  # never dereferenced: the size check runs before any launch
    # batch * heads * (d_v + 1) * 4 bytes exceeds the fixed array even with one split per (batch, head)
    assert lib.sdpa_decode_noalloc(P, P, P, P, P, None, 256, 128, 1, 128, 128, 0.1, None) == 4  # SDPA_ERR_WORKSPACE
    assert lib.sdpa_decode_noalloc(P, P, P, P, P, None, 1, 1, 16, 96, 96, 0.1, None) == 2      # SDPA_ERR_UNSUPPORTED


def test_noalloc_decode_workload_lengthens_splits_and_matches_oracle(lib, cuda_device):
    import torch
    w = W.CFG5  # 64 sequences x 32 heads, cache 16384, lengths U{1024..16384}, d = 128
    static_bytes = 16 << 20  # SDPA_DECODE_STATIC_SCRATCH_BYTES
    # at sdpa_decode's own split length the partials would overflow the fixed array, so the
    # no-alloc call must take its longer-split branch
    assert lib.sdpa_decode_workspace_size(w.batch, w.heads, w.n_cap, w.d) > static_bytes
    lens = w.lengths()
    tl = torch.from_numpy(lens).to(cuda_device)
    shape = (w.batch, w.heads, w.n_cap, w.d)
    tk = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    tv = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    si.fill_device_cache(tk, tl, w.seed, si.STREAM_K)  # rows past each length are NaN
    si.fill_device_cache(tv, tl, w.seed, si.STREAM_V)
    q = si.fill_host((w.batch, w.heads, w.d), w.seed, si.STREAM_Q)
    tq = W.to_torch(q, cuda_device)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for _ in range(2):  # two calls in a row on the shared array
        o = torch.full((w.batch, w.heads, w.d), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        l = torch.full((w.batch, w.heads), float("nan"), dtype=torch.float32, device=cuda_device)
        assert lib.sdpa_decode_noalloc(_p(tq), _p(tk), _p(tv), _p(tl), _p(o), _p(l), w.batch, w.heads, w.n_cap, w.d,
                                       w.d, w.scale_f32, st) == 0
        assert lib.sdpa_get_last_device_error(st) == 0
        outs.append((o.float().cpu().numpy().reshape(-1, w.d), l.cpu().numpy().reshape(-1)))
    # the workspace entry point on the same inputs, every (batch, head)
    need = lib.sdpa_decode_workspace_size(w.batch, w.heads, w.n_cap, w.d)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    o_ref = torch.empty((w.batch, w.heads, w.d), dtype=torch.bfloat16, device=cuda_device)
    l_ref = torch.empty((w.batch, w.heads), dtype=torch.float32, device=cuda_device)
    assert lib.sdpa_decode(_p(tq), _p(tk), _p(tv), _p(tl), _p(o_ref), _p(l_ref), w.batch, w.heads, w.n_cap, w.d, w.d,
                           w.scale_f32, _p(ws), need, st) == 0
    O_ws, L_ws = o_ref.float().cpu().numpy().reshape(-1, w.d), l_ref.cpu().numpy().reshape(-1)
    del tk, tv, ws
    torch.cuda.empty_cache()
    O, L = outs[0]
    assert np.array_equal(outs[1][0], O) and np.array_equal(outs[1][1], L)  # same inputs, same answer
    assert np.isfinite(O).all()
    assert (np.abs(O - O_ws) <= BF16_ATOL + BF16_RTOL * np.abs(O_ws)).all()
    assert np.abs(L - L_ws).max() <= LSE_TOL
    # against the oracle on sampled (batch, head) pairs, the shortest and longest sequences included
    b_min, b_max = int(np.argmin(lens)), int(np.argmax(lens))
    picks = {b_min * w.heads, b_max * w.heads + w.heads - 1}
    picks |= set(int(x) for x in si.sample_rows(w.batch * w.heads, 24, w.seed, salt=77))
    qf = si.bf16_bits_to_f32(q).reshape(-1, w.d)
    for bh in sorted(picks):
        b, h = divmod(bh, w.heads)
        n = int(lens[b])
        start = ((b * w.heads + h) * w.n_cap) * w.d
        kf = si.bf16_bits_to_f32(si.fill_host((n, w.d), w.seed, si.STREAM_K, start=start))
        vf = si.bf16_bits_to_f32(si.fill_host((n, w.d), w.seed, si.STREAM_V, start=start))
        O_ref, L_ref = oracle.sdpa_rows(qf[bh][None], kf, vf, w.scale_f32)
        err = np.abs(O[bh] - O_ref[0])
        assert (err <= BF16_ATOL + BF16_RTOL * np.abs(O_ref[0])).all(), "b=%d h=%d len=%d: max err %g" % (
            b, h, n, err.max())
        assert abs(L[bh] - L_ref[0]) <= LSE_TOL
    # a small call afterwards still matches the workspace decode (the array keeps stale partials)
    g = np.random.default_rng(5)
    _decode_both(lib, cuda_device, 3, 5, 700, 64, g.integers(1, 701, size=3).astype(np.int32), seed=23)
