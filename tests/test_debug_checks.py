"""Debug build (-DSDPA_DEBUG=1): device-side consistency checks, the stand-in for a race checker.

In this build every tensor-core kernel checks that its TMEM allocation came back
at lane 0, column 0, and the prefill kernel checks at teardown that every
pipeline barrier completed exactly as many phases (mod 2) as the roles that
use it counted -- an arrive too many or too few anywhere shows up as
SDPA_ERR_DEVICE_CHECK.  These tests run the debug library through the C ABI on
shapes that exercise every barrier path (many units per CTA, ragged tails, tiles
with no keys, windows, both head dims) and require no device error and the
oracle's answer.
"""
import ctypes
import math
import os
import subprocess

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs import workloads as W

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BF16_ATOL, BF16_RTOL, LSE_TOL = 1e-2, 1e-2, 1e-3
SDPA_ERR_DEVICE_CHECK = 8


@pytest.fixture(scope="module")
def dbg(tmp_path_factory, cuda_device):
    import importlib.util
    spec = importlib.util.spec_from_file_location("_b", os.path.join(ROOT, "memory_optimal_sdpa_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    out = str(tmp_path_factory.mktemp("debuglib") / "libsdpa_debug.so")
    subprocess.check_call(["nvcc", *b.NVCC_FLAGS, "-DSDPA_DEBUG=1", "-I", os.path.join(ROOT, "include"),
                           os.path.join(b.CSRC, "sdpa_api.cu"), "-o", out])
    L = ctypes.CDLL(out)
    _vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.sdpa_fwd.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _vp]
    L.sdpa_fwd_window.argtypes = [_vp] * 5 + [_i] * 6 + [_f, _i, _i, _vp]
    L.sdpa_bwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _vp, _sz, _vp]
    L.sdpa_bwd_workspace_size.argtypes = [_i, _i, _i]
    L.sdpa_bwd_workspace_size.restype = _sz
    L.sdpa_decode_gqa.argtypes = [_vp] * 6 + [_i] * 6 + [_f, _vp, _sz, _vp]
    L.sdpa_decode_gqa_workspace_size.argtypes = [_i] * 5
    L.sdpa_decode_gqa_workspace_size.restype = _sz
    L.sdpa_get_last_device_error.argtypes = [_vp]
    return L


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _st():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


PREFILL = [
    # (B, H, n_q, n_kv, d, mode): 0 full, 1 causal, (left, right) window
    (1, 2, 128, 128, 64, 0), (2, 3, 257, 300, 64, 1), (1, 2, 300, 100, 128, 1), (4, 40, 384, 384, 64, 1),
    (2, 80, 256, 256, 128, 0), (1, 3, 1000, 1000, 128, 1), (1, 2, 700, 700, 64, (100, 0)),
    (1, 3, 600, 900, 128, (200, 50)), (1, 150, 129, 257, 64, 0),
]


@pytest.mark.parametrize("B,H,n_q,n_kv,d,mode", PREFILL)
def test_debug_prefill_passes_its_checks(dbg, cuda_device, B, H, n_q, n_kv, d, mode):
    import torch
    seed = 300 + n_q + n_kv + d + H
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    scale = float(np.float32(1 / math.sqrt(d)))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    o = torch.full((B, H, n_q, d), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((B, H, n_q), float("nan"), dtype=torch.float32, device=cuda_device)
    for _ in range(2):  # twice: the second call starts from the barriers' fresh state again
        if isinstance(mode, tuple):
            rc = dbg.sdpa_fwd_window(_p(tq), _p(tk), _p(tv), _p(o), _p(lse), B, H, n_q, n_kv, d, d, scale, mode[0],
                                     mode[1], _st())
        else:
            rc = dbg.sdpa_fwd(_p(tq), _p(tk), _p(tv), _p(o), _p(lse), B, H, n_q, n_kv, d, d, scale, mode, _st())
        assert rc == 0
        assert dbg.sdpa_get_last_device_error(_st()) == 0
    qf, kf, vf = (si.bf16_bits_to_f32(x) for x in (q, k, v))
    if isinstance(mode, tuple):
        O_ref, L_ref = oracle.sdpa_rows_window(qf, kf, vf, scale, mode[0], mode[1])
    else:
        O_ref, L_ref = oracle.sdpa_rows(qf, kf, vf, scale, bool(mode))
    O = o.float().cpu().numpy()
    assert (np.abs(O - O_ref) <= BF16_ATOL + BF16_RTOL * np.abs(O_ref)).all()
    L = lse.cpu().numpy()
    fin = np.isfinite(L_ref)
    assert (np.isneginf(L) == ~fin).all() and np.abs(L[fin] - L_ref[fin]).max() <= LSE_TOL


@pytest.mark.parametrize("d,causal", [(64, True), (128, False)])
def test_debug_backward_passes_its_checks(dbg, cuda_device, d, causal):
    import torch
    B, H, n = 1, 3, 333
    q, k, v, do = (si.fill_host((B, H, n, d), 77 + d, s_) for s_ in (0, 1, 2, si.STREAM_DO))
    scale = float(np.float32(1 / math.sqrt(d)))
    tq, tk, tv, tdo = (W.to_torch(x, cuda_device) for x in (q, k, v, do))
    o = torch.empty_like(tq)
    lse = torch.empty((B, H, n), dtype=torch.float32, device=cuda_device)
    assert dbg.sdpa_fwd(_p(tq), _p(tk), _p(tv), _p(o), _p(lse), B, H, n, n, d, d, scale, int(causal), _st()) == 0
    dq, dk, dv = torch.empty_like(tq), torch.empty_like(tk), torch.empty_like(tv)
    need = dbg.sdpa_bwd_workspace_size(B, H, n)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    assert dbg.sdpa_bwd(_p(tq), _p(tk), _p(tv), _p(o), _p(tdo), _p(lse), _p(dq), _p(dk), _p(dv), B, H, n, n, d, d,
                        scale, int(causal), _p(ws), need, _st()) == 0
    assert dbg.sdpa_get_last_device_error(_st()) == 0
    refs = oracle.sdpa_backward(*(si.bf16_bits_to_f32(x) for x in (q, k, v, do)), scale, causal)
    for g, r in zip((dq, dk, dv), refs):
        g = g.float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(g - r) <= 1e-2 * np.linalg.norm(r)


def test_debug_grouped_decode_passes_its_checks(dbg, cuda_device):
    import torch
    B, Hq, Hkv, cap, d = 3, 32, 4, 3000, 128
    lens = np.array([3000, 1, 1777], np.int32)
    q = si.fill_host((B, Hq, d), 9, 0)
    k = si.fill_host((B, Hkv, cap, d), 9, 1)
    v = si.fill_host((B, Hkv, cap, d), 9, 2)
    scale = float(np.float32(1 / math.sqrt(d)))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    tl = torch.from_numpy(lens).to(cuda_device)
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=cuda_device)
    need = dbg.sdpa_decode_gqa_workspace_size(B, Hq, Hkv, cap, d)
    ws = torch.empty(need, dtype=torch.uint8, device=cuda_device)
    assert dbg.sdpa_decode_gqa(_p(tq), _p(tk), _p(tv), _p(tl), _p(o), _p(lse), B, Hq, Hkv, cap, d, d, scale, _p(ws),
                               need, _st()) == 0
    assert dbg.sdpa_get_last_device_error(_st()) == 0
    O_ref, _ = oracle.decode_gqa(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), lens, scale)
    O = o.float().cpu().numpy().reshape(-1, d)
    assert (np.abs(O - O_ref) <= BF16_ATOL + BF16_RTOL * np.abs(O_ref)).all()
