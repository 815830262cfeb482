"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Tolerances: bf16 outputs |O - O_ref| <= 1e-2 + 1e-2 |O_ref| elementwise; fp32
path |O - O_ref| <= 1e-5 |O_ref| + 1e-6; LSE within 1e-3 (natural-log units,
absolute) for bf16 and 1e-5 for fp32; rows that see no key must give O = 0
and LSE = -inf exactly.  Small cases compare every output against the oracle;
the full-size workloads, run through the same call the benchmark times,
compare seeded samples of query rows (or (batch, head) pairs for decode).
"""
import math

import numpy as np
import pytest

import oracle
import seeded_inputs as si
from seeded_inputs import workloads as W

pytestmark = pytest.mark.gpu

BF16_ATOL, BF16_RTOL, LSE_TOL = 1e-2, 1e-2, 1e-3


@pytest.fixture(scope="module")
def sdpa(cuda_device):
    import memory_optimal_sdpa_b200 as m
    return m


def _bits_to_torch(bits, device, pad_nan=0):
    """bf16 bits -> CUDA bf16 tensor, placed at the start of a buffer whose `pad_nan` trailing elements are NaN."""
    import torch
    flat = torch.full((bits.size + pad_nan,), float("nan"), dtype=torch.bfloat16, device=device)
    flat[:bits.size] = torch.from_numpy(bits.reshape(-1).view(np.int16)).to(device).view(torch.bfloat16)
    return flat, flat[:bits.size].view(bits.shape)


def _nan_buffer(shape, dtype, device, pad):
    import torch
    n = int(np.prod(shape))
    flat = torch.full((n + pad,), float("nan"), dtype=dtype, device=device)
    return flat, flat[:n].view(shape)


def check_bf16(O, O_ref, L, L_ref, what):
    O = O.astype(np.float64)
    err = np.abs(O - O_ref)
    bound = BF16_ATOL + BF16_RTOL * np.abs(O_ref)
    bad = ~(err <= bound)
    assert not bad.any(), "%s: %d/%d outputs out of bound, worst excess %.3g at %s" % (
        what, bad.sum(), bad.size, np.nanmax(err - bound), np.unravel_index(np.argmax(np.where(bad, err - bound, -1)), bad.shape))
    check_lse(L, L_ref, LSE_TOL, what)


def check_lse(L, L_ref, tol, what):
    L = L.astype(np.float64)
    masked = np.isneginf(L_ref)
    assert (np.isneginf(L) == masked).all(), what + ": -inf LSE pattern differs"
    d = np.abs(L[~masked] - L_ref[~masked])
    assert (d <= tol).all(), "%s: LSE max err %.3g" % (what, d.max())


# ----------------------------------------------------------------------------- bf16 prefill, small, every row
SMALL = [
    # (batch, heads, n_q, n_kv, d, causal)
    (1, 2, 128, 128, 64, False), (1, 2, 128, 128, 64, True),
    (1, 2, 128, 128, 128, False), (1, 2, 128, 128, 128, True),
    (2, 3, 257, 257, 64, True), (1, 3, 1000, 1000, 128, True), (1, 3, 1000, 1000, 64, False),
    (1, 2, 1, 1, 64, False), (1, 2, 1, 1, 128, True), (1, 2, 2, 129, 128, True), (1, 3, 127, 255, 64, True),
    (1, 2, 255, 2, 64, False), (1, 2, 300, 100, 128, True), (1, 1, 129, 1, 64, False),
    (2, 2, 512, 384, 128, False), (1, 3, 600, 1000, 64, True), (1, 1, 513, 777, 128, True),
    (3, 1, 256, 512, 64, False),
]


@pytest.mark.parametrize("B,H,n_q,n_kv,d,causal", SMALL)
def test_prefill_bf16_small(sdpa, cuda_device, B, H, n_q, n_kv, d, causal):
    import torch
    seed = hash((B, H, n_q, n_kv, d, causal)) & 0xFFFF
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    scale = float(np.float32(1 / math.sqrt(d)))
    pad = 128 * d
    _, tq = _bits_to_torch(q, cuda_device, pad)
    _, tk = _bits_to_torch(k, cuda_device, pad)
    _, tv = _bits_to_torch(v, cuda_device, pad)
    o_flat, o = _nan_buffer((B, H, n_q, d), torch.bfloat16, cuda_device, pad)
    l_flat, lse = _nan_buffer((B, H, n_q), torch.float32, cuda_device, 256)
    sdpa.fwd(tq, tk, tv, causal=causal, scale=scale, o=o, lse=lse)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.sdpa_rows(si.bf16_bits_to_f32(q), si.bf16_bits_to_f32(k), si.bf16_bits_to_f32(v), scale, causal)
    check_bf16(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref, "prefill %s" % ((B, H, n_q, n_kv, d, causal),))
    # guard bands after the outputs are untouched
    assert torch.isnan(o_flat[o.numel():]).all() and torch.isnan(l_flat[lse.numel():]).all()
    # fully masked rows (causal, n_q > n_kv): exactly zero output
    if causal and n_q > n_kv:
        O = o.float().cpu().numpy()
        assert (O[:, :, :n_q - n_kv] == 0).all()


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_causal_first_row_is_exact(sdpa, cuda_device, d):
    # Causal row 0 (n_q = n_kv) sees key 0 alone: P = 1 exactly, so O[0] = V[0] bit for bit
    # and LSE[0] = scale q_0 . k_0.  Any reference maximum above the row's true maximum (a
    # score the row may not see, or a stray value) makes P < 1 and shows here.
    import torch
    B, H, n = 2, 8, 256
    for seed in range(6):
        q, k, v = (si.fill_host((B, H, n, d), 100 + seed, s_) for s_ in (0, 1, 2))
        scale = float(np.float32(1 / math.sqrt(d)))
        o, lse = sdpa.fwd(*(W.to_torch(x, cuda_device) for x in (q, k, v)), causal=True, scale=scale)
        torch.cuda.synchronize()
        O = o.float().cpu().numpy()
        V = si.bf16_bits_to_f32(v)
        assert np.array_equal(O[:, :, 0], V[:, :, 0]), "seed %d: row 0 differs from V[0] in %d places" % (
            seed, int((O[:, :, 0] != V[:, :, 0]).sum()))
        s00 = np.einsum("bhd,bhd->bh", si.bf16_bits_to_f32(q)[:, :, 0].astype(np.float64),
                        si.bf16_bits_to_f32(k)[:, :, 0].astype(np.float64)) * scale
        assert np.abs(lse.cpu().numpy()[:, :, 0] - s00).max() < 1e-5


def test_prefill_identity_values_give_probabilities(sdpa, cuda_device):
    # V = I (n_kv = d): O = P row by row, so every probability the kernel forms is visible;
    # each entry is within two bf16 roundings (P, then O) of the exact softmax.
    import torch
    for d in (64, 128):
        for causal in (False, True):
            q, k = (si.fill_host((1, 2, d, d), 31, s_) for s_ in (0, 1))
            v = np.broadcast_to(np.eye(d, dtype=np.float32), (1, 2, d, d)).copy()
            scale = float(np.float32(1 / math.sqrt(d)))
            o, _ = sdpa.fwd(*(W.to_torch(x, cuda_device) for x in (q, k)),
                            torch.from_numpy(v).to(cuda_device).to(torch.bfloat16), causal=causal, scale=scale)
            P, _ = oracle.sdpa_rows(si.bf16_bits_to_f32(q), si.bf16_bits_to_f32(k), v, scale, causal)
            O = o.float().cpu().numpy()
            assert (np.abs(O - P) <= 2 ** -7 * P + 1e-6).all(), "d=%d causal=%d" % (d, causal)


ANY_SCALE = [
    # (n_q, n_kv, d, mode): mode full, causal, or a (left, right) window
    (256, 256, 64, "full"), (300, 333, 64, "causal"), (513, 700, 128, "causal"), (640, 640, 128, "full"),
    (333, 300, 128, "causal"), (700, 700, 64, (100, 0)), (600, 600, 128, (200, 50)),
]


@pytest.mark.parametrize("scale", [0.0, -0.125, -0.0883883461356163, -1.5])
@pytest.mark.parametrize("n_q,n_kv,d,mode", ANY_SCALE)
def test_prefill_zero_and_negative_scale(sdpa, cuda_device, n_q, n_kv, d, mode, scale):
    # The definition fixes the scale only by convention (MoA article, "DNF derivation"), so any
    # finite value is accepted: 0 gives the mean of the visible V rows and LSE = ln(count); a
    # negative scale is carried by the S product itself (negated A operand).  -1.5 drives the
    # logits far past the lazy-rescale threshold, so the running maximum moves too.
    import torch
    B, H = 1, 2
    seed = 700 + n_q + 5 * n_kv + d
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    scale = float(np.float32(scale))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    o_flat, o = _nan_buffer((B, H, n_q, d), torch.bfloat16, cuda_device, 128 * d)
    l_flat, lse = _nan_buffer((B, H, n_q), torch.float32, cuda_device, 256)
    qf, kf, vf = (si.bf16_bits_to_f32(x) for x in (q, k, v))
    if isinstance(mode, tuple):
        sdpa.fwd_window(tq, tk, tv, mode[0], mode[1], scale=scale, o=o, lse=lse)
        O_ref, L_ref = oracle.sdpa_rows_window(qf, kf, vf, scale, mode[0], mode[1])
    else:
        sdpa.fwd(tq, tk, tv, causal=(mode == "causal"), scale=scale, o=o, lse=lse)
        O_ref, L_ref = oracle.sdpa_rows(qf, kf, vf, scale, mode == "causal")
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    check_bf16(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref,
               "scale %g %s" % (scale, (n_q, n_kv, d, mode)))
    assert torch.isnan(o_flat[o.numel():]).all() and torch.isnan(l_flat[lse.numel():]).all()
    if scale == 0.0 and mode == "full":  # closed form: every row is the mean of V, LSE = ln(n_kv)
        assert np.abs(lse.cpu().numpy() - math.log(n_kv)).max() <= 1e-5


@pytest.mark.parametrize("d,causal", [(64, False), (64, True), (128, False), (128, True)])
def test_prefill_rescale_every_tile(sdpa, cuda_device, d, causal):
    # Keys grow tile by tile (128-key tiles), so every row's maximum rises by far more than the
    # lazy threshold (2^8) at each tile: the running sum and O are rescaled at every step.
    import torch
    B, H, n = 1, 2, 640
    g = np.random.default_rng(40 + d)
    q = np.abs(g.standard_normal((B, H, n, d))).astype(np.float32) * 0.25 + 0.5
    k = g.standard_normal((B, H, n, d)).astype(np.float32) * 0.05 + (np.arange(n) // 128)[None, None, :, None] * 1.25
    v = g.standard_normal((B, H, n, d)).astype(np.float32)
    to = lambda a: torch.from_numpy(a).to(cuda_device).to(torch.bfloat16)
    tq, tk, tv = to(q), to(k), to(v)
    scale = float(np.float32(1 / math.sqrt(d)))
    o, lse = sdpa.fwd(tq, tk, tv, causal=causal, scale=scale)
    qf, kf, vf = (t.float().cpu().numpy() for t in (tq, tk, tv))  # the bf16 values the kernel saw
    O_ref, L_ref = oracle.sdpa_rows(qf, kf, vf, scale, causal)
    check_bf16(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref, "rescale d=%d causal=%d" % (d, causal))
    # the logits really climb past the threshold between tiles
    s = np.einsum("d,kd->k", qf[0, 0, -1].astype(np.float64), kf[0, 0].astype(np.float64)) * scale / math.log(2)
    tile_max = s.reshape(-1, 128).max(axis=1)
    assert (np.diff(tile_max) > 8).all()


@pytest.mark.parametrize("d,mode", [(64, "full"), (64, "causal"), (128, "full"), (128, "causal"), (128, "window")])
def test_prefill_many_units_per_cta(sdpa, cuda_device, d, mode):
    # 96 (batch, head) slices of 384 rows = 192 work units of two query tiles (the second one
    # ragged): more units than SMs, so CTAs run several units back to back and every hand-over
    # between units (Q reload, O read-out, barrier phases) is checked on every row.
    import torch
    B, H, n = 8, 12, 384
    q, k, v = (si.fill_host((B, H, n, d), 60 + d, s_) for s_ in (0, 1, 2))
    scale = float(np.float32(1 / math.sqrt(d)))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    if mode == "window":
        o, lse = sdpa.fwd_window(tq, tk, tv, 100, 0, scale=scale)
        O_ref, L_ref = oracle.sdpa_rows_window(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), scale, 100, 0)
    else:
        o, lse = sdpa.fwd(tq, tk, tv, causal=(mode == "causal"), scale=scale)
        O_ref, L_ref = oracle.sdpa_rows(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), scale, mode == "causal")
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    check_bf16(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref, "many units d=%d %s" % (d, mode))


def test_prefill_lse_optional_and_repeatable(sdpa, cuda_device):
    import torch
    B, H, n, d = 1, 4, 384, 128
    q, k, v = (W.to_torch(si.fill_host((B, H, n, d), 7, s), cuda_device) for s in (0, 1, 2))
    o1, l1 = sdpa.fwd(q, k, v, causal=True)
    o2, _ = sdpa.fwd(q, k, v, causal=True, want_lse=False)
    o3, l3 = sdpa.fwd(q, k, v, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(o1, o3) and torch.equal(l1, l3)


def test_prefill_shift_invariance_on_gpu(sdpa, cuda_device):
    # K' = K + 1 u^T adds scale*(q_i . u) to row i's logits: O unchanged, LSE shifted (exact in bf16 for small ints)
    import torch
    B, H, n, d = 1, 2, 256, 64
    g = np.random.default_rng(3)
    qf = g.integers(-2, 3, (B, H, n, d)).astype(np.float32)
    kf = g.integers(-2, 3, (B, H, n, d)).astype(np.float32)
    u = g.integers(-2, 3, (d,)).astype(np.float32)
    vf = si.bf16_bits_to_f32(si.fill_host((B, H, n, d), 1, 2))
    to = lambda a: torch.from_numpy(a).to(cuda_device).to(torch.bfloat16)
    o1, l1 = sdpa.fwd(to(qf), to(kf), to(vf), scale=0.125)
    o2, l2 = sdpa.fwd(to(qf), to(kf + u), to(vf), scale=0.125)
    shift = 0.125 * np.einsum("bhnd,d->bhn", qf.astype(np.float64), u.astype(np.float64))
    np.testing.assert_allclose(o2.float().cpu().numpy(), o1.float().cpu().numpy(), atol=2e-2, rtol=2e-2)
    np.testing.assert_allclose(l2.cpu().numpy(), l1.cpu().numpy() + shift, atol=2e-3, rtol=0)


# ------------------------------------------------------------------ bf16 prefill, full-size workloads, sampled rows
def _sampled_prefill(sdpa, device, w, rows_per_head):
    import torch
    host = W.prefill_host(w)
    tq, tk, tv = (W.to_torch(host[n], device) for n in ("q", "k", "v"))
    o, lse = sdpa.fwd(tq, tk, tv, causal=w.causal, scale=w.scale_f32)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    del tq, tk, tv, o, lse
    torch.cuda.empty_cache()
    qf, kf, vf = (W.as_f32(host[n]) for n in ("q", "k", "v"))
    for b in range(w.batch):
        for h in range(w.heads):
            rows = si.sample_rows(w.n_q, rows_per_head, w.seed, salt=b * w.heads + h)
            O_ref, L_ref = oracle.sdpa_rows(qf[b, h], kf[b, h], vf[b, h], w.scale_f32, w.causal, rows=rows)
            check_bf16(O[b, h, rows], O_ref, L[b, h, rows], L_ref, "%s b=%d h=%d" % (w.name, b, h))


def test_cfg2_noncausal_sampled(sdpa, cuda_device):
    _sampled_prefill(sdpa, cuda_device, W.CFG2, 64)


def test_cfg2_causal_sampled(sdpa, cuda_device):
    _sampled_prefill(sdpa, cuda_device, W.CFG2C, 64)


def test_cfg3_causal_sampled(sdpa, cuda_device):
    _sampled_prefill(sdpa, cuda_device, W.CFG3, 256)


def test_cfg4_long_sampled(sdpa, cuda_device):
    _sampled_prefill(sdpa, cuda_device, W.CFG4, 256)


@pytest.mark.parametrize("d,causal", [(64, True), (128, False)])
def test_prefill_long_sequence_sampled(sdpa, cuda_device, d, causal):
    # n = 131072: four times cfg4's sequence (8.8 TFLOP of tile work at d = 128), one head; the
    # first, last and seeded interior rows against the oracle
    import torch
    n = 131072
    w = W.Prefill("long%d" % d, 1, 1, n, n, d, causal, "bf16", 1 / d ** 0.5)
    host = W.prefill_host(w)
    tq, tk, tv = (W.to_torch(host[x], cuda_device) for x in ("q", "k", "v"))
    o, lse = sdpa.fwd(tq, tk, tv, causal=causal, scale=w.scale_f32)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    rows = si.sample_rows(n, 48, 0, salt=d)
    O = o[0, 0, rows].float().cpu().numpy()
    L = lse[0, 0, rows].cpu().numpy()
    del tq, tk, tv, o, lse
    torch.cuda.empty_cache()
    O_ref, L_ref = oracle.sdpa_rows(*(W.as_f32(host[x])[0, 0] for x in ("q", "k", "v")), w.scale_f32, causal,
                                    rows=rows)
    check_bf16(O, O_ref, L, L_ref, "n=%d d=%d causal=%d" % (n, d, causal))


# ------------------------------------------------------------------------------------- local windows (bf16)
WINDOW_CASES = [
    # (B, H, n_q, n_kv, d, left, right)
    (1, 2, 300, 300, 64, 0, 0), (1, 2, 300, 300, 64, 5, 0), (1, 2, 600, 600, 128, 127, 0),
    (1, 2, 600, 600, 64, 128, 0), (1, 3, 1000, 1000, 128, 300, 0), (1, 2, 512, 512, 64, 64, 64),
    (1, 2, 400, 400, 128, -1, 5), (1, 2, 400, 400, 64, 200, -1), (1, 2, 257, 513, 128, 100, 0),
    (1, 2, 513, 257, 64, 100, 0), (2, 2, 384, 384, 128, -1, 0), (1, 2, 384, 384, 64, -1, -1),
    (1, 1, 700, 700, 64, 255, 255), (1, 2, 384, 384, 64, 5000, 0), (1, 2, 384, 512, 128, 5000, 5000),
]


@pytest.mark.parametrize("B,H,n_q,n_kv,d,left,right", WINDOW_CASES)
def test_prefill_window_small(sdpa, cuda_device, B, H, n_q, n_kv, d, left, right):
    import torch
    seed = 1000 + n_q + 7 * n_kv + 13 * d + left
    q = si.fill_host((B, H, n_q, d), seed, 0)
    k = si.fill_host((B, H, n_kv, d), seed, 1)
    v = si.fill_host((B, H, n_kv, d), seed, 2)
    scale = float(np.float32(1 / math.sqrt(d)))
    _, tq = _bits_to_torch(q, cuda_device, 128 * d)
    _, tk = _bits_to_torch(k, cuda_device, 128 * d)
    _, tv = _bits_to_torch(v, cuda_device, 128 * d)
    o_flat, o = _nan_buffer((B, H, n_q, d), torch.bfloat16, cuda_device, 128 * d)
    l_flat, lse = _nan_buffer((B, H, n_q), torch.float32, cuda_device, 256)
    sdpa.fwd_window(tq, tk, tv, left, right, scale=scale, o=o, lse=lse)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.sdpa_rows_window(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), scale, left, right)
    check_bf16(o.float().cpu().numpy(), O_ref, lse.cpu().numpy(), L_ref, "window %s" % ((B, H, n_q, n_kv, d, left, right),))
    assert torch.isnan(o_flat[o.numel():]).all() and torch.isnan(l_flat[lse.numel():]).all()



def _random_window_shapes(count, seed):
    # seeded shapes: ragged lengths, both head dims, windows from a single key to wider than the
    # sequence, either side open (-1)
    rng = np.random.default_rng(seed)
    out = []
    for _ in range(count):
        n_q, n_kv = int(rng.integers(1, 700)), int(rng.integers(1, 700))
        side = lambda: int(rng.choice([-1, 0, int(rng.integers(1, 300)), 1000]))
        out.append((1, int(rng.integers(1, 4)), n_q, n_kv, int(rng.choice([64, 128])), side(), side()))
    return out


@pytest.mark.parametrize("B,H,n_q,n_kv,d,left,right", _random_window_shapes(14, 77))
def test_prefill_window_random_shapes(sdpa, cuda_device, B, H, n_q, n_kv, d, left, right):
    # the full, causal and windowed kernels all sit behind sdpa_fwd_window (open sides pick the
    # plain instantiations), so random windows cover every mask mode on ragged shapes
    test_prefill_window_small(sdpa, cuda_device, B, H, n_q, n_kv, d, left, right)

def test_window_open_sides_equal_plain_calls(sdpa, cuda_device):
    import torch
    B, H, n, d = 1, 2, 640, 128
    q, k, v = (W.to_torch(si.fill_host((B, H, n, d), 9, s_), cuda_device) for s_ in (0, 1, 2))
    for causal, (left, right) in ((False, (-1, -1)), (True, (-1, 0))):
        o1, l1 = sdpa.fwd(q, k, v, causal=causal)
        o2, l2 = sdpa.fwd_window(q, k, v, left, right)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_cfg3w_window_full_size_sampled(sdpa, cuda_device):
    import torch
    w = W.CFG3W
    host = W.prefill_host(w)
    tq, tk, tv = (W.to_torch(host[n], cuda_device) for n in ("q", "k", "v"))
    o, lse = sdpa.fwd_window(tq, tk, tv, w.window[0], w.window[1], scale=w.scale_f32)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    del tq, tk, tv, o, lse
    torch.cuda.empty_cache()
    qf, kf, vf = (W.as_f32(host[n]) for n in ("q", "k", "v"))
    for h in range(0, w.heads, 4):
        rows = si.sample_rows(w.n_q, 128, w.seed, salt=h)
        O_ref, L_ref = oracle.sdpa_rows_window(qf[0, h], kf[0, h], vf[0, h], w.scale_f32, w.window[0], w.window[1],
                                               rows=rows)
        check_bf16(O[0, h, rows], O_ref, L[0, h, rows], L_ref, "cfg3w h=%d" % h)


# ------------------------------------------------------------------------------------ grouped-query decode
GQA_CASES = [
    # (B, H_q, H_kv, n_cap, d, lens)   groups of 2 .. 32 at d = 128 take the tensor cores
    (3, 8, 4, 1000, 128, (1, 1000, 517)), (2, 16, 4, 3000, 128, (2049, 129)), (2, 16, 2, 2100, 128, (128, 2100)),
    (1, 32, 2, 700, 128, (700,)), (2, 64, 2, 400, 128, (255, 400)), (1, 24, 2, 333, 128, (333,)),
    (2, 40, 2, 260, 128, (1, 260)),
    # other shapes: the CUDA-core kernel with the same head mapping
    (1, 64, 1, 300, 128, (300,)), (2, 12, 3, 500, 64, (77, 500)), (2, 4, 4, 300, 128, (5, 300)),
]


def _to_bf16_bits(x):
    """float32 -> bf16 bit patterns, round to nearest even (NaN -> the quiet NaN 0x7FC0)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    return np.where(np.isnan(x), np.uint16(0x7FC0), r)


def _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, seed):
    q = si.fill_host((B, H_q, d), seed, 0)
    k = si.fill_host((B, H_kv, n_cap, d), seed, 1)
    v = si.fill_host((B, H_kv, n_cap, d), seed, 2)
    for b in range(B):  # rows past the length hold NaN: any use of them poisons O
        k[b, :, lens[b]:] = 0x7FC0
        v[b, :, lens[b]:] = 0x7FC0
    return q, k, v


@pytest.mark.parametrize("B,H_q,H_kv,n_cap,d,lens", GQA_CASES)
def test_decode_gqa_small_every_pair(sdpa, cuda_device, B, H_q, H_kv, n_cap, d, lens):
    import torch
    lens = np.array(lens, np.int32)
    q, k, v = _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, 11 + H_q + n_cap)
    scale = float(np.float32(1 / math.sqrt(d)))
    _, tq = _bits_to_torch(q, cuda_device)
    tk, tv = (W.to_torch(x, cuda_device) for x in (k, v))
    tl = torch.from_numpy(lens).to(cuda_device)
    o_flat, o = _nan_buffer((B, H_q, d), torch.bfloat16, cuda_device, 256)
    l_flat, lse = _nan_buffer((B, H_q), torch.float32, cuda_device, 64)
    sdpa.decode_gqa(tq, tk, tv, tl, scale=scale, o=o, lse=lse)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.decode_gqa(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), lens, scale)
    check_bf16(o.float().cpu().numpy().reshape(B * H_q, d), O_ref, lse.cpu().numpy().reshape(-1), L_ref,
               "gqa %s" % ((B, H_q, H_kv, n_cap, d, tuple(lens)),))
    assert torch.isnan(o_flat[o.numel():]).all() and torch.isnan(l_flat[lse.numel():]).all()


def test_decode_gqa_many_units_per_cta(sdpa, cuda_device):
    # 48 x 16 key/value heads, one split each of one or two 128-key tiles: 768 units for the
    # persistent CTAs (several per CTA), lengths from 1 to the full cache, every pair checked
    import torch
    B, H_q, H_kv, n_cap, d = 48, 64, 16, 256, 128
    lens = si.kv_lengths(B, 1, n_cap, 77)
    lens[:3] = (1, 128, 129)
    q, k, v = _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, 77)
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    tl = torch.from_numpy(lens).to(cuda_device)
    o, lse = sdpa.decode_gqa(tq, tk, tv, tl, scale=0.09)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.decode_gqa(*(si.bf16_bits_to_f32(x) for x in (q, k, v)), lens, 0.09)
    check_bf16(o.float().cpu().numpy().reshape(B * H_q, d), O_ref, lse.cpu().numpy().reshape(-1), L_ref,
               "gqa many units")


def test_decode_gqa_long_cache(sdpa, cuda_device):
    # a 65536-row cache (four times cfg5g's), groups of 8: one sequence at full length, one short
    import torch
    B, H_q, H_kv, n_cap, d = 2, 16, 2, 65536, 128
    lens = np.array([n_cap, 3000], np.int32)
    tl = torch.from_numpy(lens).to(cuda_device)
    tk = torch.empty((B, H_kv, n_cap, d), dtype=torch.bfloat16, device=cuda_device)
    tv = torch.empty_like(tk)
    si.fill_device_cache(tk, tl, 5, si.STREAM_K)
    si.fill_device_cache(tv, tl, 5, si.STREAM_V)
    q = si.fill_host((B, H_q, d), 5, si.STREAM_Q)
    o, lse = sdpa.decode_gqa(W.to_torch(q, cuda_device), tk, tv, tl, scale=0.0884)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    G = H_q // H_kv
    for b in range(B):
        for kvh in range(H_kv):
            n = int(lens[b])
            start = ((b * H_kv + kvh) * n_cap) * d
            kf = si.bf16_bits_to_f32(si.fill_host((1, 1, n, d), 5, si.STREAM_K, start=start))
            vf = si.bf16_bits_to_f32(si.fill_host((1, 1, n, d), 5, si.STREAM_V, start=start))
            hs = slice(kvh * G, kvh * G + G)
            O_ref, L_ref = oracle.decode_gqa(si.bf16_bits_to_f32(q[b:b + 1, hs]), kf, vf, np.array([n], np.int32),
                                             0.0884)
            check_bf16(O[b, hs], O_ref, L[b, hs], L_ref, "long cache b=%d kv head %d" % (b, kvh))


def test_decode_gqa_group_of_one_is_decode(sdpa, cuda_device):
    import torch
    B, H, n_cap, d = 2, 4, 600, 128
    lens = np.array([600, 37], np.int32)
    q, k, v = _gqa_inputs(B, H, H, n_cap, d, lens, 3)
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    tl = torch.from_numpy(lens).to(cuda_device)
    o1, l1 = sdpa.decode_gqa(tq, tk, tv, tl)
    o2, l2 = sdpa.decode(tq, tk, tv, tl)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _gqa_medium(sdpa, device, q, k, v, lens, scale, what, n_groups=24):
    """A cache large enough for several 128-key tiles per split; seeded (batch, group) samples."""
    import torch
    B, H_q, d = q.shape
    H_kv, n_cap = k.shape[1], k.shape[2]
    G = H_q // H_kv
    tl = torch.from_numpy(lens).to(device)
    o, lse = sdpa.decode_gqa(W.to_torch(q, device), W.to_torch(k, device), W.to_torch(v, device), tl, scale=scale)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    for bg in sorted(set(int(x) for x in si.sample_rows(B * H_kv, n_groups, 7, salt=5))):
        b, kvh = divmod(bg, H_kv)
        n = int(lens[b])
        hs = slice(kvh * G, kvh * G + G)
        O_ref, L_ref = oracle.decode_gqa(si.bf16_bits_to_f32(q[b:b + 1, hs]), si.bf16_bits_to_f32(k[b:b + 1, kvh:kvh + 1]),
                                         si.bf16_bits_to_f32(v[b:b + 1, kvh:kvh + 1]), np.array([n], np.int32), scale)
        check_bf16(O[b, hs], O_ref, L[b, hs], L_ref, "%s b=%d kv head %d len=%d" % (what, b, kvh, n))


def test_decode_gqa_multi_tile_splits(sdpa, cuda_device):
    # 32 x 2 key/value heads x 8192 rows: 512-key splits, four 128-key tiles each
    B, H_q, H_kv, n_cap, d = 32, 16, 2, 8192, 128
    assert sdpa.decode_gqa_workspace_size(B, H_q, H_kv, n_cap, d) == B * H_q * (n_cap // 512) * (d + 1) * 4
    lens = si.kv_lengths(B, 1, n_cap, 21)
    lens[:4] = (1, 511, 513, n_cap)
    q, k, v = _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, 21)
    _gqa_medium(sdpa, cuda_device, q, k, v, lens, float(np.float32(1 / math.sqrt(d))), "gqa multi-tile")


def test_decode_gqa_zero_scale(sdpa, cuda_device):
    # scale 0: every query head of a group gets the mean of its sequence's visible value rows
    B, H_q, H_kv, n_cap, d = 4, 16, 2, 3000, 128
    lens = np.array([1, 3000, 1500, 129], np.int32)
    q, k, v = _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, 31)
    _gqa_medium(sdpa, cuda_device, q, k, v, lens, 0.0, "gqa scale 0")


def test_decode_gqa_rescale_inside_a_split(sdpa, cuda_device):
    # Scores that climb by ~12 (log2 units) from one 128-key tile to the next move every
    # head's reference maximum inside a split; a negative scale is accepted here too.
    B, H_q, H_kv, n_cap, d = 32, 16, 2, 8192, 128
    lens = np.full(B, n_cap, np.int32)
    lens[1::2] = si.kv_lengths(B // 2, 600, n_cap, 4)
    q, k, v = _gqa_inputs(B, H_q, H_kv, n_cap, d, lens, 4)
    qf = np.abs(si.bf16_bits_to_f32(q)) * 0.25 + 0.5
    kf = si.bf16_bits_to_f32(k) * 0.05 + ((np.arange(n_cap) // 128) % 4 * 0.75)[None, None, :, None]
    for sign in (1.0, -1.0):
        q2 = _to_bf16_bits(qf)
        k2 = _to_bf16_bits(kf)
        _gqa_medium(sdpa, cuda_device, q2, k2, v, lens, sign * float(np.float32(1 / math.sqrt(d))),
                    "gqa rescale sign %+d" % sign, n_groups=12)


def test_cfg5g_decode_full_size_sampled(sdpa, cuda_device):
    import torch
    w = W.CFG5G
    G = w.heads // w.kv_heads
    lens = w.lengths()
    tl = torch.from_numpy(lens).to(cuda_device)
    shape = (w.batch, w.kv_heads, w.n_cap, w.d)
    tk = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    tv = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    si.fill_device_cache(tk, tl, w.seed, si.STREAM_K)
    si.fill_device_cache(tv, tl, w.seed, si.STREAM_V)
    q = si.fill_host((w.batch, w.heads, w.d), w.seed, si.STREAM_Q)
    o, lse = sdpa.decode_gqa(W.to_torch(q, cuda_device), tk, tv, tl, scale=w.scale_f32)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy()
    L = lse.cpu().numpy()
    del tk, tv
    torch.cuda.empty_cache()
    # (batch, key/value head) groups: the shortest and the longest sequence, plus seeded picks
    b_min, b_max = int(np.argmin(lens)), int(np.argmax(lens))
    picks = {b_min * w.kv_heads, b_max * w.kv_heads + w.kv_heads - 1}
    picks |= set(int(x) for x in si.sample_rows(w.batch * w.kv_heads, 30, w.seed, salt=98))
    for bg in sorted(picks):
        b, kvh = divmod(bg, w.kv_heads)
        n = int(lens[b])
        start = ((b * w.kv_heads + kvh) * w.n_cap) * w.d
        kf = si.bf16_bits_to_f32(si.fill_host((1, 1, n, w.d), w.seed, si.STREAM_K, start=start))
        vf = si.bf16_bits_to_f32(si.fill_host((1, 1, n, w.d), w.seed, si.STREAM_V, start=start))
        hs = slice(kvh * G, kvh * G + G)
        O_ref, L_ref = oracle.decode_gqa(si.bf16_bits_to_f32(q[b:b + 1, hs]), kf, vf, np.array([n], np.int32),
                                         w.scale_f32)
        check_bf16(O[b, hs], O_ref, L[b, hs], L_ref, "cfg5g b=%d kv head %d len=%d" % (b, kvh, n))


# ----------------------------------------------------------------------------------------------- fp32 path
F32_CASES = [(1, 1, 128, 128, 64, 64, False), (1, 1, 128, 128, 64, 64, True), (2, 3, 77, 130, 33, 100, True),
             (1, 2, 200, 50, 128, 128, True), (1, 1, 1, 1, 1, 1, False), (1, 2, 65, 300, 3, 128, False)]


@pytest.mark.parametrize("B,H,n_q,n_kv,dk,dv,causal", F32_CASES)
def test_prefill_f32(sdpa, cuda_device, B, H, n_q, n_kv, dk, dv, causal):
    q = si.fill_host((B, H, n_q, dk), 0, 0, bf16=False)
    k = si.fill_host((B, H, n_kv, dk), 0, 1, bf16=False)
    v = si.fill_host((B, H, n_kv, dv), 0, 2, bf16=False)
    scale = float(np.float32(1 / math.sqrt(dk)))
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    o, lse = sdpa.fwd_f32(tq, tk, tv, causal=causal, scale=scale)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.sdpa_rows(q, k, v, scale, causal)
    O = o.cpu().numpy().astype(np.float64)
    err = np.abs(O - O_ref)
    assert (err <= 1e-5 * np.abs(O_ref) + 1e-6).all(), "max rel err %.3g" % (err / (np.abs(O_ref) + 1e-6)).max()
    check_lse(lse.cpu().numpy(), L_ref, 1e-5, "f32")


@pytest.mark.parametrize("scale", [0.0, -0.125, -0.0883883461356163])
@pytest.mark.parametrize("causal", [False, True])
def test_prefill_f32_zero_and_negative_scale(sdpa, cuda_device, causal, scale):
    # any finite scale on the CUDA-core path too: 0 gives the mean of the visible rows, a negative
    # scale flips the logits (rows 0.. of a causal call see 1.. keys).  Scales of the fp32
    # workload's magnitude: the 1e-5 relative bound holds for logits of that size (at |scale| = 1
    # the fp32 rounding of the 64-term dot products alone, about |s| 2^-24 sqrt(d), exceeds it).
    B, H, n_q, n_kv, d = 1, 2, 150, 170, 64
    q = si.fill_host((B, H, n_q, d), 8, 0, bf16=False)
    k = si.fill_host((B, H, n_kv, d), 8, 1, bf16=False)
    v = si.fill_host((B, H, n_kv, d), 8, 2, bf16=False)
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    o, lse = sdpa.fwd_f32(tq, tk, tv, causal=causal, scale=scale)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.sdpa_rows(q, k, v, scale, causal)
    err = np.abs(o.cpu().numpy().astype(np.float64) - O_ref)
    assert (err <= 1e-5 * np.abs(O_ref) + 1e-6).all(), "scale %g: max err %.3g" % (scale, err.max())
    check_lse(lse.cpu().numpy(), L_ref, 1e-5, "f32 scale %g" % scale)


def test_cfg1_fp32(sdpa, cuda_device):
    w = W.CFG1
    host = W.prefill_host(w)
    tq, tk, tv = (W.to_torch(host[n], cuda_device) for n in ("q", "k", "v"))
    o, lse = sdpa.fwd_f32(tq, tk, tv, causal=w.causal, scale=w.scale_f32)
    O_ref, L_ref = oracle.sdpa_rows(host["q"], host["k"], host["v"], w.scale_f32, w.causal)
    O = o.cpu().numpy().astype(np.float64)
    assert (np.abs(O - O_ref) <= 1e-5 * np.abs(O_ref) + 1e-6).all()
    check_lse(lse.cpu().numpy(), L_ref, 1e-5, "cfg1")


# -------------------------------------------------------------------------------------------------- decode
@pytest.mark.parametrize("scale_kind", ["default", "zero", "negative"])
@pytest.mark.parametrize("d", [64, 128])
def test_decode_small_every_pair(sdpa, cuda_device, d, scale_kind):
    import torch
    B, H, n_cap = 3, 4, 1000
    lens = np.array([1, 1000, 517], np.int32)
    q = si.fill_host((B, H, d), 5, 0)
    k = si.fill_host((B, H, n_cap, d), 5, 1)
    v = si.fill_host((B, H, n_cap, d), 5, 2)
    for b in range(B):  # rows past the length hold NaN: any read of them poisons O
        k[b, :, lens[b]:] = 0x7FC0
        v[b, :, lens[b]:] = 0x7FC0
    # any finite scale: 0 averages the visible rows, a negative one flips the logits
    scale = {"default": float(np.float32(1 / math.sqrt(d))), "zero": 0.0, "negative": -0.25}[scale_kind]
    tq, tk, tv = (W.to_torch(x, cuda_device) for x in (q, k, v))
    tl = torch.from_numpy(lens).to(cuda_device)
    o, lse = sdpa.decode(tq, tk, tv, tl, scale=scale)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O_ref, L_ref = oracle.decode(si.bf16_bits_to_f32(q), si.bf16_bits_to_f32(k), si.bf16_bits_to_f32(v), lens, scale)
    check_bf16(o.float().cpu().numpy().reshape(B * H, d), O_ref, lse.cpu().numpy().reshape(-1), L_ref,
               "decode d=%d scale %g" % (d, scale))


def test_decode_bad_length_reported(sdpa, cuda_device):
    import torch
    B, H, n_cap, d = 2, 2, 64, 64
    tq = torch.zeros((B, H, d), dtype=torch.bfloat16, device=cuda_device)
    tk = torch.zeros((B, H, n_cap, d), dtype=torch.bfloat16, device=cuda_device)
    tl = torch.tensor([5, 65], dtype=torch.int32, device=cuda_device)
    sdpa.decode(tq, tk, tk, tl)
    assert sdpa.get_last_device_error() == sdpa.SDPA_ERR_DEVICE_BAD_LENGTH
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK  # read clears the word


def test_cfg5_decode_full_size_sampled(sdpa, cuda_device):
    import torch
    w = W.CFG5
    lens = w.lengths()
    tl = torch.from_numpy(lens).to(cuda_device)
    shape = (w.batch, w.heads, w.n_cap, w.d)
    tk = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    tv = torch.empty(shape, dtype=torch.bfloat16, device=cuda_device)
    si.fill_device_cache(tk, tl, w.seed, si.STREAM_K)
    si.fill_device_cache(tv, tl, w.seed, si.STREAM_V)
    q = si.fill_host((w.batch, w.heads, w.d), w.seed, si.STREAM_Q)
    o, lse = sdpa.decode(W.to_torch(q, cuda_device), tk, tv, tl, scale=w.scale_f32)
    assert sdpa.get_last_device_error() == sdpa.SDPA_OK
    O = o.float().cpu().numpy().reshape(-1, w.d)
    L = lse.cpu().numpy().reshape(-1)
    del tk, tv
    torch.cuda.empty_cache()
    # pairs: both heads 0 and H-1 of the shortest and the longest sequence, plus seeded picks
    b_min, b_max = int(np.argmin(lens)), int(np.argmax(lens))
    picks = {b_min * w.heads, b_min * w.heads + w.heads - 1, b_max * w.heads, b_max * w.heads + w.heads - 1}
    picks |= set(int(x) for x in si.sample_rows(w.batch * w.heads, 60, w.seed, salt=99))
    qf = si.bf16_bits_to_f32(q).reshape(-1, w.d)
    for bh in sorted(picks):
        b, h = divmod(bh, w.heads)
        n = int(lens[b])
        start = ((b * w.heads + h) * w.n_cap) * w.d
        kf = si.bf16_bits_to_f32(si.fill_host((n, w.d), w.seed, si.STREAM_K, start=start))
        vf = si.bf16_bits_to_f32(si.fill_host((n, w.d), w.seed, si.STREAM_V, start=start))
        O_ref, L_ref = oracle.sdpa_rows(qf[bh][None], kf, vf, w.scale_f32)
        check_bf16(O[bh][None], O_ref, L[bh:bh + 1], L_ref, "cfg5 b=%d h=%d len=%d" % (b, h, n))
