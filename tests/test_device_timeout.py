"""Failure detection without a GPU fault: a pipeline wait that runs out reports an error and the GPU stays usable.

A test-only build of the library (SDPA_FAULT_DROP_ARRIVE, 20 ms wait budget) has
softmax warpgroup b skip its first "P ready" arrive, so the MMA issuer of that
tile waits on a barrier phase nothing will complete.  Every pipeline wait in the
kernel is time-bounded: the waiting thread sets the CTA's abort flag and the
device error word, the other roles leave their loops, copies and MMAs in flight
are drained, TMEM is released and the kernel returns.  The host reads
SDPA_ERR_DEVICE_TIMEOUT, and a normal call on the same context still gives the
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


@pytest.fixture(scope="module")
def fault_lib(tmp_path_factory, cuda_device):
    import importlib.util
    spec = importlib.util.spec_from_file_location("_b", os.path.join(ROOT, "memory_optimal_sdpa_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    out = str(tmp_path_factory.mktemp("faultlib") / "libsdpa_fault.so")
    subprocess.check_call(["nvcc", *b.NVCC_FLAGS, "-DSDPA_FAULT_DROP_ARRIVE", "-DSDPA_WAIT_BUDGET_NS=20000000ull",
                           "-I", os.path.join(ROOT, "include"), os.path.join(b.CSRC, "sdpa_api.cu"), "-o", out])
    L = ctypes.CDLL(out)
    _vp, _i, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.sdpa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
    L.sdpa_get_last_device_error.argtypes = [_vp]
    return L


def test_timeout_is_reported_and_context_survives(fault_lib, cuda_device):
    import torch
    import memory_optimal_sdpa_b200 as sdpa
    B, H, n, d = 1, 2, 256, 64
    q, k, v = (si.fill_host((B, H, n, d), 4, s) for s in (0, 1, 2))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    o = torch.zeros((B, H, n, d), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.zeros((B, H, n), dtype=torch.float32, device=cuda_device)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    for _ in range(2):  # the failure is reported every time, never as a sticky CUDA error
        assert fault_lib.sdpa_fwd(P(tq), P(tk), P(tv), P(o), P(lse), B, H, n, n, d, d, 0.125, 0, st) == 0
        assert fault_lib.sdpa_get_last_device_error(st) == sdpa.SDPA_ERR_DEVICE_TIMEOUT
    torch.cuda.synchronize()  # no CUDA error on the context
    # the production library on the same context: correct results, no device error
    o2, l2 = sdpa.fwd(tq, tk, tv, scale=0.125)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.sdpa_rows(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), 0.125, False)
    err = np.abs(o2.float().cpu().numpy() - O_ref)
    assert (err <= 1e-2 + 1e-2 * np.abs(O_ref)).all()
    assert np.abs(l2.cpu().numpy() - L_ref).max() <= 1e-3
