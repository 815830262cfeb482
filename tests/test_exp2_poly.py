"""The prefill kernel's FMA-pipe exponential (sm100::exp2_poly2), checked on the GPU.

At d = 64 one column pair in eight of every unmasked key tile takes its
exponentials from a polynomial on the FMA pipe instead of the MUFU unit.  Two
checks pin it:
  - directly: a test-only probe kernel evaluates exp2_poly2 (and exp2f) on a dense
    grid of [-125, 8], the range the softmax feeds it (x = s*c - m <= 0, up to 8
    above the stale maximum under lazy rescaling), and both are compared with the
    exact 2^x in double: relative error <= 1e-4;
  - in use: with V = [I; 0] and V = [0; I] over one unmasked 128-key tile, O is the
    probability row itself, so every probability the polynomial forms (columns
    14-15, 30-31, ...) is visible and must be within two bf16 roundings of the
    oracle's softmax.
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
def probe(tmp_path_factory, cuda_device):
    out = str(tmp_path_factory.mktemp("exp2probe") / "libexp2probe.so")
    subprocess.check_call(["nvcc", "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-shared",
                           "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "memory_optimal_sdpa_b200", "csrc"),
                           os.path.join(ROOT, "tests", "exp2_poly_probe.cu"), "-o", out])
    L = ctypes.CDLL(out)
    L.exp2_poly_eval.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int, ctypes.c_void_p]
    return L


def test_exp2_poly_relative_error(probe, cuda_device):
    import torch
    grid = np.linspace(-125.0, 8.0, 1 << 21, dtype=np.float64)
    special = np.array([-125.0, -124.5, -1.5, -1.0, -0.5, -0.25, 0.0, 0.25, 0.5, 1.0, 7.5, 8.0,
                        np.nextafter(np.float32(-0.5), np.float32(0)), np.nextafter(np.float32(0.5), np.float32(1))])
    x = np.concatenate([grid, special]).astype(np.float32)
    if x.size % 2:
        x = np.append(x, np.float32(-3.0))
    tx = torch.from_numpy(x).to(cuda_device)
    yp, yl = torch.empty_like(tx), torch.empty_like(tx)
    st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert probe.exp2_poly_eval(ctypes.c_void_p(tx.data_ptr()), ctypes.c_void_p(yp.data_ptr()),
                                ctypes.c_void_p(yl.data_ptr()), x.size // 2, st) == 0
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    rel_poly = np.abs(yp.cpu().numpy().astype(np.float64) / exact - 1)
    rel_lib = np.abs(yl.cpu().numpy().astype(np.float64) / exact - 1)
    worst = int(np.argmax(rel_poly))
    assert rel_poly.max() <= 1e-4, "exp2_poly2: relative error %.3g at x = %r" % (rel_poly.max(), float(x[worst]))
    assert rel_lib.max() <= 1e-6  # the comparison itself is sound: exp2f is accurate on this range
    # and against the device's own exp2f, as used elsewhere
    assert (np.abs(yp.cpu().numpy().astype(np.float64) - yl.cpu().numpy()) <= 1e-4 * exact).all()
    # integer inputs are exact powers of two up to the polynomial's error at f = 0
    ints = np.arange(-125, 9, dtype=np.float32)
    sel = np.isin(x, ints)
    assert sel.sum() >= 10
    assert (rel_poly[sel] <= 1e-4).all()


def test_prefill_unmasked_tile_probabilities(cuda_device):
    # One unmasked 128-key tile at d = 64 (non-causal, n_kv = 128): with V = [I; 0], O holds
    # P[:, 0:64]; with V = [0; I], P[:, 64:128].  Two query tiles, two heads, two seeds.
    import torch
    import memory_optimal_sdpa_b200 as sdpa
    d, n_q, n_kv = 64, 256, 128
    eye = np.eye(d, dtype=np.float32)
    zero = np.zeros((d, d), np.float32)
    for seed in (41, 42):
        q, k = (si.fill_host((1, 2, n, d), seed, s_) for s_, n in ((0, n_q), (1, n_kv)))
        scale = float(np.float32(1 / math.sqrt(d)))
        tq, tk = (W.to_torch(x, cuda_device) for x in (q, k))
        qf, kf = si.bf16_bits_to_f32(q), si.bf16_bits_to_f32(k)
        for half, v2 in ((0, np.concatenate([eye, zero])), (1, np.concatenate([zero, eye]))):
            v = np.broadcast_to(v2, (1, 2, n_kv, d)).copy()
            o, _ = sdpa.fwd(tq, tk, torch.from_numpy(v).to(cuda_device).to(torch.bfloat16), scale=scale)
            assert sdpa.get_last_device_error() == sdpa.SDPA_OK
            P, _ = oracle.sdpa_rows(qf, kf, v, scale, False)  # = the probability columns of this half
            O = o.float().cpu().numpy()
            bad = ~(np.abs(O - P) <= 2 ** -7 * P + 1e-6)
            assert not bad.any(), "seed %d half %d: %d probabilities off, columns %s" % (
                seed, half, bad.sum(), sorted(set((np.nonzero(bad)[-1] + 64 * half).tolist()))[:16])
            # the rows' probabilities over both halves sum to 1 (checked on the oracle side once)
            if half == 1:
                full = np.concatenate([P_prev, P], axis=-1)
                assert np.allclose(full.sum(-1), 1.0, atol=1e-12)
            P_prev = P
