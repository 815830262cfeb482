"""Pins for the CPU oracle: checks against facts fixed by the definition, not by the oracle itself.

The method is exact attention, Attention(Q,K,V) = softmax(Q K^T * scale) V with
a numerically stable (max-subtracted) softmax, derived with no intermediate
arrays ("Attention at the Theoretical Minimum: A Mathematics of Arrays
Framework for Memory-Optimal Transformer Kernels", abstract; agents-report.net
MoA article, sections "DNF derivation" and "numerical verification").  The
pages print no worked numbers, so the pins are closed forms, invariants,
special cases that reduce to a library routine, and brute force.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(12345)


def _frac(s):
    return float(Fraction(s))


def _ln(s):
    assert s.startswith("ln ")
    return math.log(float(s[3:]))


@pytest.mark.parametrize("causal", [False, True])
def test_worked_example_closed_form(causal):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    q = np.array(g["Q"], np.float32)
    k = np.array(g["K"], np.float32)
    v = np.array(g["V"], np.float32)
    exp = g["causal" if causal else "noncausal"]
    O_exp = np.array([[_frac(x) for x in row] for row in exp["O"]])
    L_exp = np.array([_ln(x) for x in exp["LSE"]])
    for O, L in (oracle.sdpa_rows(q, k, v, math.log(2.0), causal), oracle.sdpa_full(q, k, v, math.log(2.0), causal)[:2]):
        np.testing.assert_allclose(O, O_exp, rtol=0, atol=1e-15)
        np.testing.assert_allclose(L, L_exp, rtol=0, atol=1e-15)
    # the score matrix itself: scale * Q K^T, not K Q^T
    S = oracle.scores(q, k, math.log(2.0), causal)
    dots = np.array(g["dots"], np.float64) * math.log(2.0)
    if causal:
        dots[0, 2] = -np.inf
    np.testing.assert_array_equal(S, dots)


def test_single_key_returns_v_exactly():
    # n_kv = 1: the only weight is exp(0)/exp(0) = 1, so O = V[0] bit for bit and LSE = s_00.
    q = RNG.integers(-4, 5, size=(6, 16)).astype(np.float32)
    k = RNG.integers(-4, 5, size=(1, 16)).astype(np.float32)
    v = RNG.standard_normal((1, 8)).astype(np.float32)
    O, L = oracle.sdpa_rows(q, k, v, 0.25)
    np.testing.assert_array_equal(O, np.broadcast_to(v.astype(np.float64), O.shape))
    dots = (q.astype(np.int64) @ k.astype(np.int64).T)[:, 0]  # exact integer dot products
    np.testing.assert_array_equal(L, 0.25 * dots.astype(np.float64))


def test_causal_first_row_is_v0():
    n, d = 9, 8
    q, k, v = (RNG.standard_normal((n, d)).astype(np.float32) for _ in range(3))
    O, L = oracle.sdpa_rows(q, k, v, 0.3, causal=True)
    np.testing.assert_array_equal(O[0], v[0].astype(np.float64))
    S = oracle.scores(q[:1], k[:1], 0.3)
    assert L[0] == S[0, 0]


def test_constant_v_gives_constant_output():
    n_q, n_kv, d = 7, 11, 5
    q, k = RNG.standard_normal((n_q, d)).astype(np.float32), RNG.standard_normal((n_kv, d)).astype(np.float32)
    row = RNG.standard_normal(6).astype(np.float32)
    v = np.tile(row, (n_kv, 1))
    for causal in (False, True):
        O, _ = oracle.sdpa_rows(q, k, v, 0.7, causal)
        np.testing.assert_allclose(O, np.broadcast_to(row.astype(np.float64), O.shape), rtol=4e-16, atol=0)


def test_softmax_rows_sum_to_one_and_identity_v():
    n, d = 12, 12
    q, k = RNG.standard_normal((n, 8)).astype(np.float32), RNG.standard_normal((n, 8)).astype(np.float32)
    for causal in (False, True):
        S = oracle.scores(q, k, 0.9, causal)
        P = oracle.softmax_rows(S)
        np.testing.assert_allclose(P.sum(1), 1.0, rtol=0, atol=1e-15)
        assert (P >= 0).all()
        # V = I (n_kv = d_v) turns the output into the probability matrix itself
        O, _ = oracle.sdpa_rows(q, k, np.eye(n, d, dtype=np.float32), 0.9, causal)
        np.testing.assert_allclose(O, P, rtol=0, atol=1e-15)
        np.testing.assert_allclose(O.sum(1), 1.0, rtol=0, atol=1e-15)
        if causal:
            assert (O[np.triu_indices(n, 1)] == 0).all()


@pytest.mark.parametrize("causal", [False, True])
def test_zero_logits_give_mean_of_allowed_rows(causal):
    n_q, n_kv, d = 6, 9, 4
    q = RNG.standard_normal((n_q, d)).astype(np.float32)
    k = RNG.standard_normal((n_kv, d)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 5)).astype(np.float32)
    for qq, scale in ((np.zeros_like(q), 0.5), (q, 0.0)):
        O, L = oracle.sdpa_rows(qq, k, v, scale, causal)
        for i in range(n_q):
            cnt = (i + n_kv - n_q + 1) if causal else n_kv
            np.testing.assert_allclose(O[i], v[:cnt].astype(np.float64).mean(0), rtol=1e-14, atol=1e-15)
            assert abs(L[i] - math.log(cnt)) < 1e-15


def test_permutation_equivariance():
    n_q, n_kv, d = 5, 13, 8
    q = RNG.standard_normal((n_q, d)).astype(np.float32)
    k = RNG.standard_normal((n_kv, d)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 6)).astype(np.float32)
    O, L = oracle.sdpa_rows(q, k, v, 0.4)
    perm = RNG.permutation(n_kv)
    O2, L2 = oracle.sdpa_rows(q, k[perm], v[perm], 0.4)
    np.testing.assert_allclose(O2, O, rtol=0, atol=1e-14)
    np.testing.assert_allclose(L2, L, rtol=0, atol=1e-14)
    # permuting V alone must change the answer (the pairing of k_j with v_j matters)
    O3, _ = oracle.sdpa_rows(q, k, v[perm], 0.4)
    assert np.abs(O3 - O).max() > 1e-3


def test_shift_invariance():
    # K' = K + 1 u^T adds scale*(q_i . u) to every logit of row i: O unchanged, LSE shifted.
    n_q, n_kv, d = 4, 10, 8
    q = RNG.integers(-3, 4, size=(n_q, d)).astype(np.float32)
    k = RNG.integers(-3, 4, size=(n_kv, d)).astype(np.float32)
    u = RNG.integers(-5, 6, size=(d,)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 7)).astype(np.float32)
    scale = 0.125
    for causal in (False, True):
        O, L = oracle.sdpa_rows(q, k, v, scale, causal)
        O2, L2 = oracle.sdpa_rows(q, k + u, v, scale, causal)
        shift = scale * (q.astype(np.int64) @ u.astype(np.int64)).astype(np.float64)
        np.testing.assert_allclose(O2, O, rtol=0, atol=1e-13)
        np.testing.assert_allclose(L2, L + shift, rtol=0, atol=1e-12)


def _brute_force(q, k, v, scale, causal):
    """Independent pure-Python evaluation of the naive formula exp(s)/sum exp(s) (no max subtraction)."""
    n_q, n_kv = len(q), len(k)
    O, L = [], []
    for i in range(n_q):
        ws = []
        for j in range(n_kv):
            if causal and j > i + (n_kv - n_q):
                ws.append(0.0)
                continue
            s = scale * math.fsum(float(a) * float(b) for a, b in zip(q[i], k[j]))
            ws.append(math.exp(s))
        z = math.fsum(ws)
        O.append([math.fsum(w * float(v[j][c]) for j, w in enumerate(ws)) / z for c in range(len(v[0]))])
        L.append(math.log(z))
    return np.array(O), np.array(L)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_q,n_kv,d_k,d_v", [(1, 1, 1, 1), (3, 5, 4, 2), (8, 8, 6, 3), (5, 8, 2, 7)])
def test_brute_force_tiny(n_q, n_kv, d_k, d_v, causal):
    q = RNG.uniform(-1, 1, (n_q, d_k)).astype(np.float32)
    k = RNG.uniform(-1, 1, (n_kv, d_k)).astype(np.float32)
    v = RNG.standard_normal((n_kv, d_v)).astype(np.float32)
    scale = 1.3  # |s| < 5
    O, L = oracle.sdpa_rows(q, k, v, scale, causal)
    Ob, Lb = _brute_force(q, k, v, scale, causal)
    np.testing.assert_allclose(O, Ob, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(L, Lb, rtol=0, atol=1e-13)
    S = oracle.scores(q, k, scale, causal)
    np.testing.assert_allclose(oracle.softmax_rows(S), oracle.softmax_naive(S), rtol=1e-13, atol=1e-15)


def test_stability_large_logits():
    # s = [800, 799, 798]: exp(800) overflows, the max-subtracted form gives weights 1 : e^-1 : e^-2.
    q = np.array([[1.0]], np.float32)
    k = np.array([[800.0], [799.0], [798.0]], np.float32)
    v = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]], np.float32)
    with np.errstate(over="ignore", invalid="ignore"):
        naive = oracle.softmax_naive(oracle.scores(q, k, 1.0))
    assert not np.isfinite(naive).all()
    O, L = oracle.sdpa_rows(q, k, v, 1.0)
    z = 1 + math.exp(-1) + math.exp(-2)
    np.testing.assert_allclose(O[0], [(1 + math.exp(-2)) / z, (math.exp(-1) + math.exp(-2)) / z], rtol=1e-15)
    assert abs(L[0] - (800 + math.log(z))) < 1e-12


def test_causal_alignment_rectangular():
    # bottom-right alignment: row i sees keys j <= i + (n_kv - n_q)
    d = 4
    q = RNG.standard_normal((3, d)).astype(np.float32)
    k = RNG.standard_normal((2, d)).astype(np.float32)
    v = RNG.standard_normal((2, 3)).astype(np.float32)
    O, L = oracle.sdpa_rows(q, k, v, 0.5, causal=True)
    assert (O[0] == 0).all() and L[0] == -np.inf          # no allowed key
    np.testing.assert_array_equal(O[1], v[0].astype(np.float64))  # only key 0
    Of, Lf = oracle.sdpa_rows(q, k, v, 0.5, causal=False)
    np.testing.assert_allclose(O[2], Of[2], rtol=0, atol=1e-15)   # last row sees everything
    # a single query row (decode) is unaffected by the causal flag
    k5 = RNG.standard_normal((5, d)).astype(np.float32)
    v5 = RNG.standard_normal((5, 3)).astype(np.float32)
    a = oracle.sdpa_rows(q[:1], k5, v5, 0.5, causal=True)
    b = oracle.sdpa_rows(q[:1], k5, v5, 0.5, causal=False)
    np.testing.assert_array_equal(a[0], b[0])


@pytest.mark.parametrize("causal", [False, True])
def test_library_special_case_torch_float64(causal):
    # Mirrors the pages' check of the DNF against PyTorch in double precision.
    import torch
    import seeded_inputs as si
    n, d = 128, 64
    q, k, v = (si.fill_host((1, 1, n, d), 0, s, bf16=False) for s in (0, 1, 2))
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(x).double() for x in (q, k, v)), is_causal=causal, scale=1 / 8).numpy()
    O, _ = oracle.sdpa_rows(q, k, v, 1 / 8, causal)
    np.testing.assert_allclose(O, ref, rtol=1e-12, atol=1e-13)


def test_rows_subset_and_slices_match_full():
    bh, n_q, n_kv, d = 3, 20, 17, 8
    q = RNG.standard_normal((bh, n_q, d)).astype(np.float32)
    k = RNG.standard_normal((bh, n_kv, d)).astype(np.float32)
    v = RNG.standard_normal((bh, n_kv, 5)).astype(np.float32)
    rows = np.array([0, 3, 19, 7])
    for causal in (False, True):
        O, L = oracle.sdpa_rows(q, k, v, 0.3, causal, rows=rows, threads=3)
        for b in range(bh):
            Of, Lf, _, _ = oracle.sdpa_full(q[b], k[b], v[b], 0.3, causal)
            np.testing.assert_allclose(O[b], Of[rows], rtol=1e-14, atol=1e-15)
            np.testing.assert_allclose(L[b], Lf[rows], rtol=1e-14, atol=1e-15)


def test_decode_uses_only_first_len_keys():
    B, H, n_cap, d = 3, 2, 16, 8
    q = RNG.standard_normal((B, H, d)).astype(np.float32)
    k = RNG.standard_normal((B, H, n_cap, d)).astype(np.float32)
    v = RNG.standard_normal((B, H, n_cap, d)).astype(np.float32)
    lens = np.array([1, 16, 7], np.int32)
    for b in range(B):
        k[b, :, lens[b]:] = np.nan
        v[b, :, lens[b]:] = np.nan
    O, L = oracle.decode(q, k, v, lens, 0.35)
    assert np.isfinite(O).all() and np.isfinite(L).all()
    for b in range(B):
        for h in range(H):
            n = lens[b]
            Or, Lr = oracle.sdpa_rows(q[b, h][None], k[b, h, :n], v[b, h, :n], 0.35)
            np.testing.assert_array_equal(O[b * H + h], Or[0])
            assert L[b * H + h] == Lr[0]
    np.testing.assert_array_equal(O[0], v[0, 0, 0].astype(np.float64))  # len 1 -> V[0]
    pairs = np.array([5, 0])
    Op, Lp = oracle.decode(q, k, v, lens, 0.35, pairs=pairs)
    np.testing.assert_array_equal(Op, O[pairs])


def test_rejects_bad_arguments():
    q = np.zeros((2, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.sdpa_rows(q, q, q, 1.0, rows=np.array([2]))
    with pytest.raises(ValueError):
        oracle.decode(np.zeros((1, 1, 4), np.float32), np.zeros((1, 1, 4, 4), np.float32),
                      np.zeros((1, 1, 4, 4), np.float32), np.array([5], np.int32), 1.0)


# ------------------------------------------------------------------------------------------- local windows
# Sliding (local) windows generalise the causal mask: row i, at key position p = i + (n_kv - n_q),
# sees keys p - left <= j <= p + right (the windowed attention the 2-simplicial article uses to
# bound cost, applied here to ordinary attention).
def test_window_zero_width_returns_own_v_row():
    n_q, n_kv, d = 5, 9, 6
    q = RNG.integers(-3, 4, size=(n_q, d)).astype(np.float32)
    k = RNG.integers(-3, 4, size=(n_kv, d)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 4)).astype(np.float32)
    O, L = oracle.sdpa_rows_window(q, k, v, 0.5, 0, 0)
    for i in range(n_q):
        p = i + n_kv - n_q
        np.testing.assert_array_equal(O[i], v[p].astype(np.float64))
        assert L[i] == 0.5 * float(q[i].astype(np.int64) @ k[p].astype(np.int64))


def test_window_reduces_to_full_and_causal():
    n_q, n_kv, d = 7, 11, 5
    q, k = RNG.standard_normal((n_q, d)).astype(np.float32), RNG.standard_normal((n_kv, d)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 3)).astype(np.float32)
    for (left, right), causal in (((-1, -1), False), ((-1, 0), True), ((n_kv, n_kv), False), ((n_kv, 0), True)):
        Ow, Lw = oracle.sdpa_rows_window(q, k, v, 0.4, left, right)
        O, L = oracle.sdpa_rows(q, k, v, 0.4, causal)
        np.testing.assert_array_equal(Ow, O)
        np.testing.assert_array_equal(Lw, L)


def _brute_force_window(q, k, v, scale, left, right):
    n_q, n_kv = len(q), len(k)
    O, L = [], []
    for i in range(n_q):
        p = i + n_kv - n_q
        ws = []
        for j in range(n_kv):
            if (left >= 0 and j < p - left) or (right >= 0 and j > p + right):
                ws.append(0.0)
                continue
            ws.append(math.exp(scale * math.fsum(float(a) * float(b) for a, b in zip(q[i], k[j]))))
        z = math.fsum(ws)
        if z == 0:
            O.append([0.0] * len(v[0])); L.append(-math.inf); continue
        O.append([math.fsum(w * float(v[j][c]) for j, w in enumerate(ws)) / z for c in range(len(v[0]))])
        L.append(math.log(z))
    return np.array(O), np.array(L)


@pytest.mark.parametrize("left,right", [(0, 0), (2, 0), (3, 1), (-1, 2), (1, -1), (4, 4)])
@pytest.mark.parametrize("n_q,n_kv", [(6, 6), (4, 9), (9, 4)])
def test_window_brute_force(n_q, n_kv, left, right):
    q = RNG.uniform(-1, 1, (n_q, 4)).astype(np.float32)
    k = RNG.uniform(-1, 1, (n_kv, 4)).astype(np.float32)
    v = RNG.standard_normal((n_kv, 3)).astype(np.float32)
    O, L = oracle.sdpa_rows_window(q, k, v, 1.1, left, right)
    Ob, Lb = _brute_force_window(q, k, v, 1.1, left, right)
    np.testing.assert_allclose(O, Ob, rtol=1e-13, atol=1e-14)
    assert (np.isneginf(L) == np.isneginf(Lb)).all()
    fin = np.isfinite(Lb)
    np.testing.assert_allclose(L[fin], Lb[fin], rtol=0, atol=1e-13)


# ------------------------------------------------------------------------------------ grouped-query decode
# Query head h of H_q reads key/value head h // (H_q // H_kv): consecutive query heads share one
# key/value head (the grouped-query layout the 2-simplicial article tiles along).
def test_gqa_equals_decode_on_an_expanded_cache():
    # Replicating every key/value head over its group turns grouped-query decode into plain decode.
    B, H_q, H_kv, n_cap, d = 3, 8, 2, 11, 5
    q = RNG.standard_normal((B, H_q, d)).astype(np.float32)
    k = RNG.standard_normal((B, H_kv, n_cap, d)).astype(np.float32)
    v = RNG.standard_normal((B, H_kv, n_cap, 4)).astype(np.float32)
    lens = np.array([11, 1, 6], np.int32)
    G = H_q // H_kv
    k_exp = np.repeat(k, G, axis=1)  # head h of the expanded cache is head h // G
    v_exp = np.repeat(v, G, axis=1)
    O, L = oracle.decode_gqa(q, k, v, lens, 0.7)
    Oe, Le = oracle.decode(q, k_exp, v_exp, lens, 0.7)
    np.testing.assert_array_equal(O, Oe)
    np.testing.assert_array_equal(L, Le)


def test_gqa_group_of_one_is_decode_and_pairs_select():
    B, H, n_cap, d = 2, 3, 7, 4
    q = RNG.standard_normal((B, H, d)).astype(np.float32)
    k = RNG.standard_normal((B, H, n_cap, d)).astype(np.float32)
    v = RNG.standard_normal((B, H, n_cap, d)).astype(np.float32)
    lens = np.array([7, 3], np.int32)
    O, L = oracle.decode_gqa(q, k, v, lens, 0.5)
    Od, Ld = oracle.decode(q, k, v, lens, 0.5)
    np.testing.assert_array_equal(O, Od)
    np.testing.assert_array_equal(L, Ld)
    pairs = np.array([5, 0, 3], np.int64)
    Op, Lp = oracle.decode_gqa(q, k, v, lens, 0.5, pairs=pairs)
    np.testing.assert_array_equal(Op, O[pairs])
    np.testing.assert_array_equal(Lp, L[pairs])


def test_gqa_brute_force_and_group_closed_form():
    # Brute force in plain Python; and a group whose queries are all zero attends uniformly:
    # O = mean of the first len rows of its key/value head's V, LSE = ln len.
    B, H_q, H_kv, n_cap, d = 2, 6, 3, 5, 3
    q = RNG.uniform(-1, 1, (B, H_q, d)).astype(np.float32)
    q[1, 2:4] = 0.0  # batch 1, group 1 (query heads 2 and 3 -> key/value head 1)
    k = RNG.uniform(-1, 1, (B, H_kv, n_cap, d)).astype(np.float32)
    v = RNG.standard_normal((B, H_kv, n_cap, 2)).astype(np.float32)
    lens = np.array([5, 4], np.int32)
    O, L = oracle.decode_gqa(q, k, v, lens, 1.3)
    G = H_q // H_kv
    for b in range(B):
        for h in range(H_q):
            kv = h // G
            n = int(lens[b])
            w = [math.exp(1.3 * math.fsum(float(a) * float(c) for a, c in zip(q[b, h], k[b, kv, j])))
                 for j in range(n)]
            z = math.fsum(w)
            ref = [math.fsum(w[j] * float(v[b, kv, j, c]) for j in range(n)) / z for c in range(2)]
            np.testing.assert_allclose(O[b * H_q + h], ref, rtol=1e-13, atol=1e-14)
            assert abs(L[b * H_q + h] - math.log(z)) < 1e-13
    for h in (2, 3):
        np.testing.assert_allclose(O[1 * H_q + h], v[1, 1, :4].astype(np.float64).mean(axis=0), rtol=1e-14)
        assert abs(L[1 * H_q + h] - math.log(4)) < 1e-14


def test_gqa_rejects_bad_groups():
    with pytest.raises(ValueError):
        oracle.decode_gqa(np.zeros((1, 3, 4), np.float32), np.zeros((1, 2, 4, 4), np.float32),
                          np.zeros((1, 2, 4, 4), np.float32), np.array([4], np.int32), 1.0)


# ------------------------------------------------------------------------------------------- backward pass
# The gradients of L = sum(O * dO) for the forward definition (the MoA roadmap's last stage is
# the backward pass).  Pinned by finite differences of the forward oracle, torch float64
# autograd, and identities that hold for any inputs.
def _loss(q, k, v, do, scale, causal):
    O, _ = oracle.sdpa_rows(q, k, v, scale, causal)
    return float(np.sum(O * do.astype(np.float64)))


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_finite_differences(causal):
    n_q, n_kv, d_k, d_v = 4, 6, 3, 2
    g = np.random.default_rng(7)
    # dyadic inputs well inside float32: perturbations of +-2^-12 are exact
    q = (g.integers(-8, 9, (n_q, d_k)) / 8).astype(np.float32)
    k = (g.integers(-8, 9, (n_kv, d_k)) / 8).astype(np.float32)
    v = (g.integers(-8, 9, (n_kv, d_v)) / 8).astype(np.float32)
    do = (g.integers(-8, 9, (n_q, d_v)) / 8).astype(np.float32)
    scale, h = 0.7, 2.0 ** -12
    dQ, dK, dV = oracle.sdpa_backward(q, k, v, do, scale, causal)
    for x, grad in ((q, dQ), (k, dK), (v, dV)):
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = [xp if y is x else y for y in (q, k, v)]
            args_m = [xm if y is x else y for y in (q, k, v)]
            fd = (_loss(*args_p, do, scale, causal) - _loss(*args_m, do, scale, causal)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-7, (idx, fd, grad[idx])


@pytest.mark.parametrize("causal", [False, True])
def test_backward_matches_torch_float64_autograd(causal):
    import torch
    B, H, n_q, n_kv, d = 2, 2, 9, 13, 8
    g = np.random.default_rng(8)
    q, k, v, do = (g.standard_normal(s).astype(np.float32) for s in
                   ((B, H, n_q, d), (B, H, n_kv, d), (B, H, n_kv, d), (B, H, n_q, d)))
    scale = 0.3
    dQ, dK, dV = oracle.sdpa_backward(q, k, v, do, scale, causal)
    tq, tk, tv = (torch.from_numpy(x).double().requires_grad_(True) for x in (q, k, v))
    # bottom-right aligned causal mask written out: row i sees keys j <= i + n_kv - n_q
    mask = None
    if causal:
        mask = torch.from_numpy(np.arange(n_kv)[None, :] <= np.arange(n_q)[:, None] + (n_kv - n_q))
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask, scale=scale)
    out.backward(torch.from_numpy(do).double())
    np.testing.assert_allclose(dQ, tq.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, tv.grad.numpy(), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_identities(causal):
    # Rows of P sum to one: sum_j dV_j = sum_i dO_i (over rows that see a key).  Rows of dS sum
    # to zero: sum_j dK_j = 0.  Adding a constant row to V leaves dQ and dK unchanged.
    n_q, n_kv, d = 11, 7, 5
    q, k, do = (RNG.standard_normal(s).astype(np.float32) for s in ((n_q, d), (n_kv, d), (n_q, d)))
    v = (RNG.integers(-64, 65, (n_kv, d)) / 16).astype(np.float32)  # dyadic: v + 3 is exact
    dQ, dK, dV = oracle.sdpa_backward(q, k, v, do, 0.45, causal)
    seen = np.arange(n_q) + (n_kv - n_q) >= 0 if causal else np.ones(n_q, bool)
    np.testing.assert_allclose(dV.sum(axis=0), do[seen].astype(np.float64).sum(axis=0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dK.sum(axis=0), 0.0, atol=1e-12)
    dQ2, dK2, _ = oracle.sdpa_backward(q, k, v + np.float32(3.0), do, 0.45, causal)
    np.testing.assert_allclose(dQ2, dQ, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK2, dK, rtol=1e-10, atol=1e-12)


def test_backward_single_key_closed_form():
    # One key: P = 1 everywhere, so dV_0 = sum_i dO_i and dQ = dK = 0 exactly.
    q = RNG.standard_normal((5, 4)).astype(np.float32)
    k = RNG.standard_normal((1, 4)).astype(np.float32)
    v = RNG.standard_normal((1, 3)).astype(np.float32)
    do = RNG.standard_normal((5, 3)).astype(np.float32)
    dQ, dK, dV = oracle.sdpa_backward(q, k, v, do, 0.9)
    assert (dQ == 0).all() and (dK == 0).all()
    np.testing.assert_allclose(dV[0], do.astype(np.float64).sum(axis=0), rtol=1e-15)


def test_backward_row_selection():
    n_q, n_kv, d = 10, 12, 4
    q, k, v, do = (RNG.standard_normal(s).astype(np.float32) for s in ((n_q, d), (n_kv, d), (n_kv, d), (n_q, d)))
    dQ, dK, dV = oracle.sdpa_backward(q, k, v, do, 0.5, True)
    qr, kr = np.array([9, 0, 4]), np.array([11, 3])
    sQ, sK, sV = oracle.sdpa_backward(q, k, v, do, 0.5, True, q_rows=qr, k_rows=kr)
    np.testing.assert_array_equal(sQ, dQ[qr])
    np.testing.assert_array_equal(sK, dK[kr])
    np.testing.assert_array_equal(sV, dV[kr])
