"""GPU parity of the backward pass (sdpa_bwd through the C ABI) against the CPU oracle's gradients.

The GPU gradients start from the GPU forward's own outputs (O in bf16 and LSE), as a
caller's training step would; the oracle differentiates the exact definition in double.

Tolerance, per gradient tensor G of one (batch, head) slice:
    |G - G_ref| <= 0.03 |G_ref| + 0.03 rms(G_ref)
P and dS enter the tensor cores rounded to bf16 (relative 2^-9 each) and D_i = dO_i . O_i
uses the bf16-rounded forward output, an error shared by every key of row i; the sums over
up to n rows of such terms give errors of a few 2^-9 of the tensor's typical magnitude,
which the rms term bounds, plus the bf16 rounding of the result itself (the |G_ref| term).
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs import workloads as W

pytestmark = pytest.mark.gpu

RTOL, RMS_TOL = 0.03, 0.03


@pytest.fixture(scope="module")
def sdpa(cuda_device):
    import memory_optimal_sdpa_b200 as m
    return m


def check_grad(G, G_ref, what):
    G = G.astype(np.float64)
    rms = math.sqrt(float(np.mean(G_ref ** 2))) if G_ref.size else 0.0
    err = np.abs(G - G_ref)
    bound = RTOL * np.abs(G_ref) + RMS_TOL * rms
    bad = ~(err <= bound)
    assert not bad.any(), "%s: %d/%d out of bound (rms %.3g), worst excess %.3g at %s" % (
        what, bad.sum(), bad.size, rms, np.nanmax(err - bound),
        np.unravel_index(np.argmax(np.where(bad, err - bound, -1)), bad.shape))


def run_bwd(sdpa, device, q, k, v, do, causal, scale):
    import torch
    tq, tk, tv, tdo = (W.to_torch(x, device) for x in (q, k, v, do))
    o, lse = sdpa.fwd(tq, tk, tv, causal=causal, scale=scale)
    dq, dk, dv = sdpa.bwd(tq, tk, tv, o, tdo, lse, causal=causal, scale=scale)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    torch.cuda.synchronize()
    return tuple(x.float().cpu().numpy() for x in (dq, dk, dv))


SMALL = [
    # (B, H, n_q, n_kv, d, causal)
    (1, 2, 128, 128, 64, False), (1, 2, 128, 128, 64, True), (1, 2, 256, 256, 128, True),
    (1, 2, 300, 300, 64, True), (1, 1, 200, 333, 128, False), (1, 2, 333, 200, 64, True),
    (1, 2, 333, 200, 128, False), (2, 2, 1, 1, 128, False), (1, 2, 640, 640, 128, False),
    (1, 3, 513, 700, 64, True),
]


@pytest.mark.parametrize("B,H,n_q,n_kv,d,causal", SMALL)
def test_bwd_small_every_element(sdpa, cuda_device, B, H, n_q, n_kv, d, causal):
    seed = 500 + n_q + 3 * n_kv + d + int(causal)
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    do = si.fill_host((B, H, n_q, d), seed, si.STREAM_DO)
    scale = float(np.float32(1 / math.sqrt(d)))
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, causal, scale)
    dQ, dK, dV = oracle.sdpa_backward(*(si.bf16_bits_to_f32(x) for x in (q, k, v, do)), scale, causal)
    for b in range(B):
        for h in range(H):
            tag = "%s b=%d h=%d" % ((B, H, n_q, n_kv, d, causal), b, h)
            check_grad(dq[b, h], dQ[b, h], "dQ " + tag)
            check_grad(dk[b, h], dK[b, h], "dK " + tag)
            check_grad(dv[b, h], dV[b, h], "dV " + tag)
    if causal and n_q > n_kv:  # rows that see no key get no gradient
        assert (dq[:, :, :n_q - n_kv] == 0).all()


def test_bwd_single_key_closed_form(sdpa, cuda_device):
    # One key: P = 1, so dV_0 = sum_i dO_i and dQ = dK = 0 exactly (dP - D vanishes).
    B, H, n_q, d = 1, 2, 200, 64
    q = si.fill_host((B, H, n_q, d), 3, 0)
    k = si.fill_host((B, H, 1, d), 3, 1)
    v = si.fill_host((B, H, 1, d), 3, 2)
    do = si.fill_host((B, H, n_q, d), 3, si.STREAM_DO)
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, False, 0.125)
    ref = si.bf16_bits_to_f32(do).astype(np.float64).sum(axis=2)
    check_grad(dv[:, :, 0], ref, "dV single key")
    assert np.abs(dq).max() < 1e-2 * np.abs(si.bf16_bits_to_f32(do)).max() and np.abs(dk).max() < 1e-2


def _sampled_slices(sdpa, device, w, slices, causal):
    """Full workload on the GPU, every element of the listed (batch, head) slices checked."""
    host = W.prefill_host(w)
    do = si.fill_host((w.batch, w.heads, w.n_q, w.d), w.seed, si.STREAM_DO)
    dq, dk, dv = run_bwd(sdpa, device, host["q"], host["k"], host["v"], do, causal, w.scale_f32)
    for b, h in slices:
        qf, kf, vf = (W.as_f32(host[n][b, h]) for n in ("q", "k", "v"))
        dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, si.bf16_bits_to_f32(do[b, h]), w.scale_f32, causal)
        tag = "%s b=%d h=%d" % (w.name, b, h)
        check_grad(dq[b, h], dQ, "dQ " + tag)
        check_grad(dk[b, h], dK, "dK " + tag)
        check_grad(dv[b, h], dV, "dV " + tag)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_cfg2_full_size_four_slices(sdpa, cuda_device, causal):
    _sampled_slices(sdpa, cuda_device, W.CFG2, [(0, 0), (1, 5), (2, 10), (3, 15)], causal)


def test_bwd_d128_causal_medium(sdpa, cuda_device):
    w = W.Prefill("bwd_d128", 1, 8, 2048, 2048, 128, True, "bf16", 1 / 128 ** 0.5, v=W.Dist(si.UNIFORM, -1.0, 1.0))
    _sampled_slices(sdpa, cuda_device, w, [(0, 0), (0, 3), (0, 7)], True)
