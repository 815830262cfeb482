"""GPU parity of the backward pass (sdpa_bwd through the C ABI) against the CPU oracle's gradients.

The GPU gradients start from the GPU forward's own outputs (O in bf16 and LSE), as a
caller's training step would; the oracle differentiates the exact definition in double.

Tolerance: every element within the worst-case error of the kernels' bf16 arithmetic,
bounded term by term (numpy, float64, for the bound only -- the reference is the oracle):
P and dS enter the tensor cores rounded to bf16, and D_i = dO_i . O_i uses the forward's
bf16 O, an error delta_i <= 2^-9 sum_c |dO_ic O_ic| shared by every key of row i, so
    |dV - ref| <= 2^-8 (P^T |dO|)
    |dK - ref| <= scale ((2^-8 |dS| + P delta)^T |Q|)
    |dQ - ref| <= scale ((2^-8 |dS| + P delta) |K|)
each plus 2^-8 |ref| (the bf16 result) and 1e-5 (fp32 residue where a gradient cancels
exactly).  The roundings are counted at 2^-8, twice the half-ulp, for margin.  Each tensor
also has to agree as a whole: ||G - ref|| <= 1e-2 ||ref|| (Frobenius), which a systematic
error -- a dropped term, a wrong mask -- cannot meet.
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs import workloads as W

pytestmark = pytest.mark.gpu

ATOL, FRO_TOL = 1e-5, 1e-2


@pytest.fixture(scope="module")
def sdpa(cuda_device):
    import memory_optimal_sdpa_b200 as m
    return m


def grad_bounds(q, k, v, do, scale, causal):
    """Elementwise error bounds of the bf16 path for one slice (float32 inputs, 2-D)."""
    q, k, v, do = (x.astype(np.float64) for x in (q, k, v, do))
    n_q, n_kv = q.shape[0], k.shape[0]
    s = scale * (q @ k.T)
    if causal:
        s = np.where(np.arange(n_kv)[None, :] <= np.arange(n_q)[:, None] + (n_kv - n_q), s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    p = np.where(z > 0, e / np.where(z > 0, z, 1.0), 0.0)
    dp = do @ v.T
    o = p @ v
    ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
    delta = 2.0 ** -9 * np.abs(do * o).sum(axis=1, keepdims=True)
    w = 2.0 ** -8 * np.abs(ds) + p * delta
    a = abs(scale)
    return (a * (w @ np.abs(k)), a * (w.T @ np.abs(q)), 2.0 ** -8 * (p.T @ np.abs(do)))


def check_grad(G, G_ref, bound, what):
    G = G.astype(np.float64)
    err = np.abs(G - G_ref)
    lim = bound + 2.0 ** -8 * np.abs(G_ref) + ATOL
    bad = ~(err <= lim)
    assert not bad.any(), "%s: %d/%d out of bound, worst excess %.3g at %s" % (
        what, bad.sum(), bad.size, np.nanmax(err - lim),
        np.unravel_index(np.argmax(np.where(bad, err - lim, -1)), bad.shape))
    nref = np.linalg.norm(G_ref)
    assert np.linalg.norm(G - G_ref) <= FRO_TOL * nref + ATOL * math.sqrt(G.size), \
        "%s: relative Frobenius error %.3g" % (what, np.linalg.norm(G - G_ref) / max(nref, 1e-300))


def check_slice(dq, dk, dv, dQ, dK, dV, qf, kf, vf, dof, scale, causal, tag):
    bq, bk, bv = grad_bounds(qf, kf, vf, dof, scale, causal)
    check_grad(dq, dQ, bq, "dQ " + tag)
    check_grad(dk, dK, bk, "dK " + tag)
    check_grad(dv, dV, bv, "dV " + tag)


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
    qf, kf, vf, dof = (si.bf16_bits_to_f32(x) for x in (q, k, v, do))
    dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, scale, causal)
    for b in range(B):
        for h in range(H):
            tag = "%s b=%d h=%d" % ((B, H, n_q, n_kv, d, causal), b, h)
            check_slice(dq[b, h], dk[b, h], dv[b, h], dQ[b, h], dK[b, h], dV[b, h], qf[b, h], kf[b, h], vf[b, h],
                        dof[b, h], scale, causal, tag)
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
    err = np.abs(dv[:, :, 0] - ref)
    assert (err <= 2.0 ** -8 * np.abs(si.bf16_bits_to_f32(do)).astype(np.float64).sum(axis=2) + 2.0 ** -8 * np.abs(ref)).all()
    assert np.abs(dq).max() < 1e-4 and np.abs(dk).max() < 1e-4


def _sampled_slices(sdpa, device, w, slices, causal):
    """Full workload on the GPU, every element of the listed (batch, head) slices checked."""
    host = W.prefill_host(w)
    do = si.fill_host((w.batch, w.heads, w.n_q, w.d), w.seed, si.STREAM_DO)
    dq, dk, dv = run_bwd(sdpa, device, host["q"], host["k"], host["v"], do, causal, w.scale_f32)
    for b, h in slices:
        qf, kf, vf = (W.as_f32(host[n][b, h]) for n in ("q", "k", "v"))
        dof = si.bf16_bits_to_f32(do[b, h])
        dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, w.scale_f32, causal)
        check_slice(dq[b, h], dk[b, h], dv[b, h], dQ, dK, dV, qf, kf, vf, dof, w.scale_f32, causal,
                    "%s b=%d h=%d" % (w.name, b, h))


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_cfg2_full_size_four_slices(sdpa, cuda_device, causal):
    _sampled_slices(sdpa, cuda_device, W.CFG2, [(0, 0), (1, 5), (2, 10), (3, 15)], causal)


def test_bwd_d128_causal_medium(sdpa, cuda_device):
    w = W.Prefill("bwd_d128", 1, 8, 2048, 2048, 128, True, "bf16", 1 / 128 ** 0.5, v=W.Dist(si.UNIFORM, -1.0, 1.0))
    _sampled_slices(sdpa, cuda_device, w, [(0, 0), (0, 3), (0, 7)], True)


MANY_UNITS = [
    # (B, H, n_q, n_kv, d, causal): more 128-row units than SMs, so each persistent CTA walks
    # several units (ragged tails; the last case has query tiles that see no key)
    (2, 80, 333, 333, 64, True), (1, 160, 200, 300, 128, False), (2, 96, 300, 200, 64, False),
    (2, 80, 333, 100, 64, True), (1, 96, 640, 512, 128, True),
]


@pytest.mark.parametrize("B,H,n_q,n_kv,d,causal", MANY_UNITS)
def test_bwd_many_units_per_cta(sdpa, cuda_device, B, H, n_q, n_kv, d, causal):
    seed = 900 + n_q + n_kv + d + int(causal)
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    do = si.fill_host((B, H, n_q, d), seed, si.STREAM_DO)
    scale = float(np.float32(1 / math.sqrt(d)))
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, causal, scale)
    # every element of every 7th slice, so each CTA position in the dealing is sampled
    for i in range(0, B * H, 7):
        b, h = divmod(i, H)
        qf, kf, vf, dof = (si.bf16_bits_to_f32(x[b, h]) for x in (q, k, v, do))
        dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, scale, causal)
        check_slice(dq[b, h], dk[b, h], dv[b, h], dQ, dK, dV, qf, kf, vf, dof, scale, causal,
                    "%s b=%d h=%d" % ((B, H, n_q, n_kv, d, causal), b, h))
    if causal and n_q > n_kv:
        assert (dq[:, :, :n_q - n_kv] == 0).all()


def test_bwd_complete_for_work_queued_behind_it(sdpa, cuda_device):
    # dq runs as a programmatic dependent of dkdv (it may start on SMs dkdv's last wave leaves), so
    # the stream must still order later work after all three gradients: copies queued right behind
    # sdpa_bwd, with no synchronisation in between, must equal the gradients read after a sync.
    import torch
    w = W.CFG2
    host = W.prefill_host(w)
    q, k, v = (W.to_torch(host[n], cuda_device) for n in ("q", "k", "v"))
    do = W.to_torch(si.fill_host((w.batch, w.heads, w.n_q, w.d), w.seed, si.STREAM_DO), cuda_device)
    for causal in (False, True):
        o, lse = sdpa.fwd(q, k, v, causal=causal, scale=w.scale_f32)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        for _ in range(3):
            for g in (dq, dk, dv):
                g.zero_()
            sdpa.bwd(q, k, v, o, do, lse, causal=causal, scale=w.scale_f32, dq=dq, dk=dk, dv=dv)
            copies = [g.clone() for g in (dq, dk, dv)]  # same stream, queued behind the backward
            torch.cuda.synchronize()
            for name, c, g in zip(("dQ", "dK", "dV"), copies, (dq, dk, dv)):
                assert torch.equal(c, g), "%s read behind sdpa_bwd differs (causal=%s)" % (name, causal)
            assert dv.abs().sum().item() > 0
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK


@pytest.mark.parametrize("scale", [0.0, -0.125, -0.0883883461356163])
@pytest.mark.parametrize("B,H,n_q,n_kv,d,causal", [(1, 2, 256, 256, 64, True), (1, 2, 300, 200, 128, False),
                                                    (1, 2, 333, 333, 128, True), (1, 2, 200, 333, 64, False)])
def test_bwd_zero_and_negative_scale(sdpa, cuda_device, B, H, n_q, n_kv, d, causal, scale):
    # The gradient formulas hold for any finite scale (the MoA article's definition fixes the
    # scale only by convention): scale = 0 makes P uniform over the visible keys and dQ = dK = 0;
    # a negative scale flips the logits.  The forward feeding this is the same call.
    seed = 900 + n_q + 3 * n_kv + d + int(causal)
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    do = si.fill_host((B, H, n_q, d), seed, si.STREAM_DO)
    scale = float(np.float32(scale))
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, causal, scale)
    qf, kf, vf, dof = (si.bf16_bits_to_f32(x) for x in (q, k, v, do))
    dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, scale, causal)
    for b in range(B):
        for h in range(H):
            tag = "%s scale=%g b=%d h=%d" % ((B, H, n_q, n_kv, d, causal), scale, b, h)
            check_slice(dq[b, h], dk[b, h], dv[b, h], dQ[b, h], dK[b, h], dV[b, h], qf[b, h], kf[b, h], vf[b, h],
                        dof[b, h], scale, causal, tag)
    if scale == 0.0:
        assert (dq == 0).all() and (dk == 0).all()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("scale,std", [(1e-3, 1.0), (None, 2.5)])
def test_bwd_extreme_logit_ranges(sdpa, cuda_device, d, causal, scale, std):
    # The tensor-core backward adds -LSE log2(e) / (scale log2(e)) to S inside the S product, as
    # three bf16 terms: a tiny scale makes that term large against S (about 1e4 here), and wide
    # inputs (N(0, 2.5^2), the 1 x 8 x 32768 workload's distribution) make the softmax sharp.
    # Both must stay within the same per-element bounds as the ordinary cases.
    B, H, n = 1, 2, 320
    seed = 950 + d + int(causal) + (0 if scale is None else 7)
    q = si.fill_host((B, H, n, d), seed, 0, b=std)
    k = si.fill_host((B, H, n, d), seed, 1, b=std)
    v = si.fill_host((B, H, n, d), seed, 2)
    do = si.fill_host((B, H, n, d), seed, si.STREAM_DO)
    scale = float(np.float32(1 / math.sqrt(d) if scale is None else scale))
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, causal, scale)
    qf, kf, vf, dof = (si.bf16_bits_to_f32(x) for x in (q, k, v, do))
    dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, scale, causal)
    for h in range(H):
        check_slice(dq[0, h], dk[0, h], dv[0, h], dQ[0, h], dK[0, h], dV[0, h], qf[0, h], kf[0, h], vf[0, h],
                    dof[0, h], scale, causal, "d=%d causal=%s scale=%g std=%g h=%d" % (d, causal, scale, std, h))


def _random_shapes(count, seed):
    # seeded shapes: ragged lengths on both sides, both head dims, both masks, several heads
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(count):
        out.append((1, int(rng.integers(1, 4)), int(rng.integers(1, 600)), int(rng.integers(1, 600)),
                    int(rng.choice([64, 128])), bool(rng.integers(0, 2))))
    return out


@pytest.mark.parametrize("B,H,n_q,n_kv,d,causal", _random_shapes(12, 2024))
def test_bwd_random_shapes(sdpa, cuda_device, B, H, n_q, n_kv, d, causal):
    seed = 1300 + 7 * n_q + 3 * n_kv + d + int(causal)
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    do = si.fill_host((B, H, n_q, d), seed, si.STREAM_DO)
    scale = float(np.float32(1 / math.sqrt(d)))
    dq, dk, dv = run_bwd(sdpa, cuda_device, q, k, v, do, causal, scale)
    qf, kf, vf, dof = (si.bf16_bits_to_f32(x) for x in (q, k, v, do))
    dQ, dK, dV = oracle.sdpa_backward(qf, kf, vf, dof, scale, causal)
    for h in range(H):
        check_slice(dq[0, h], dk[0, h], dv[0, h], dQ[0, h], dK[0, h], dV[0, h], qf[0, h], kf[0, h], vf[0, h],
                    dof[0, h], scale, causal, "%s h=%d" % ((B, H, n_q, n_kv, d, causal), h))
