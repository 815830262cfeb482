"""Python access to the CPU oracle -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline and
reference legs may import this package.  The product path
(memory_optimal_sdpa_b200) never does.  See oracle.h for what is computed and
which passages of the attention pages it follows.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)


def threads_available():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def lib():
    global _lib
    if _lib is None:
        # SDPA_ORACLE_LIBRARY lets the mutation test load a deliberately broken copy.
        path = os.environ.get("SDPA_ORACLE_LIBRARY") or _build.build()
        L = ctypes.CDLL(path)
        I64, I32, D = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        L.oracle_scores.argtypes = [_f32p, _f32p, I64, I64, I32, D, I32, _f64p]
        L.oracle_softmax_rows.argtypes = [_f64p, I64, I64, _f64p]
        L.oracle_softmax_naive.argtypes = [_f64p, I64, I64, _f64p]
        L.oracle_sdpa_full.argtypes = [_f32p, _f32p, _f32p, I64, I64, I32, I32, D, I32, _f64p, _f64p,
                                       _f64p, _f64p]
        L.oracle_sdpa_rows.argtypes = [_f32p, _f32p, _f32p, I64, I64, I64, I32, I32, D, I32, _i64p, I64,
                                       _f64p, _f64p, I32]
        L.oracle_sdpa_rows_window.argtypes = [_f32p, _f32p, _f32p, I64, I64, I64, I32, I32, D, I64, I64, _i64p,
                                               I64, _f64p, _f64p, I32]
        L.oracle_sdpa_rows_window.restype = ctypes.c_int
        L.oracle_decode.argtypes = [_f32p, _f32p, _f32p, _i32p, I64, I64, I64, I32, I32, D, _i64p, I64,
                                    _f64p, _f64p, I32]
        L.oracle_decode_gqa.argtypes = [_f32p, _f32p, _f32p, _i32p, I64, I64, I64, I64, I32, I32, D, _i64p, I64,
                                        _f64p, _f64p, I32]
        L.oracle_decode_gqa.restype = ctypes.c_int
        L.oracle_sdpa_backward.argtypes = [_f32p, _f32p, _f32p, _f32p, I64, I64, I64, I32, I32, D, I32, _i64p, I64,
                                           _i64p, I64, _f64p, _f64p, _f64p, I32]
        L.oracle_sdpa_backward.restype = ctypes.c_int
        for f in (L.oracle_scores, L.oracle_softmax_rows, L.oracle_softmax_naive, L.oracle_sdpa_full,
                  L.oracle_sdpa_rows, L.oracle_decode):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _f32(a):
    a = np.ascontiguousarray(a, dtype=np.float32)
    return a, a.ctypes.data_as(_f32p)


def _check(rc, name):
    if rc != 0:
        raise ValueError("%s rejected its arguments" % name)


def scores(q, k, scale, causal=False):
    """S = scale * q k^T with masked entries at -inf; q [n_q, d_k], k [n_kv, d_k]."""
    q, qp = _f32(q)
    k, kp = _f32(k)
    S = np.empty((q.shape[0], k.shape[0]), dtype=np.float64)
    _check(lib().oracle_scores(qp, kp, q.shape[0], k.shape[0], q.shape[1], scale, int(causal),
                               S.ctypes.data_as(_f64p)), "oracle_scores")
    return S


def softmax_rows(S):
    S = np.ascontiguousarray(S, dtype=np.float64)
    P = np.empty_like(S)
    _check(lib().oracle_softmax_rows(S.ctypes.data_as(_f64p), S.shape[0], S.shape[1], P.ctypes.data_as(_f64p)),
           "oracle_softmax_rows")
    return P


def softmax_naive(S):
    S = np.ascontiguousarray(S, dtype=np.float64)
    P = np.empty_like(S)
    _check(lib().oracle_softmax_naive(S.ctypes.data_as(_f64p), S.shape[0], S.shape[1], P.ctypes.data_as(_f64p)),
           "oracle_softmax_naive")
    return P


def sdpa_full(q, k, v, scale, causal=False):
    """Full-matrix form for one slice. Returns (O, LSE, S, P)."""
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    n_q, d_k = q.shape
    n_kv, d_v = v.shape
    S = np.empty((n_q, n_kv)); P = np.empty((n_q, n_kv))
    O = np.empty((n_q, d_v)); L = np.empty((n_q,))
    _check(lib().oracle_sdpa_full(qp, kp, vp, n_q, n_kv, d_k, d_v, scale, int(causal),
                                  S.ctypes.data_as(_f64p), P.ctypes.data_as(_f64p),
                                  O.ctypes.data_as(_f64p), L.ctypes.data_as(_f64p)), "oracle_sdpa_full")
    return O, L, S, P


def sdpa_rows(q, k, v, scale, causal=False, rows=None, threads=None):
    """Row-at-a-time form over leading slice dims.

    q [..., n_q, d_k], k [..., n_kv, d_k], v [..., n_kv, d_v] (same leading dims).
    rows: None (all rows) or a 1-D array of query-row indices used for every slice.
    Returns O [..., n_rows, d_v] and LSE [..., n_rows] in float64.
    """
    lead = q.shape[:-2]
    n_q, d_k = q.shape[-2:]
    n_kv, d_v = v.shape[-2:]
    bh = int(np.prod(lead, dtype=np.int64)) if lead else 1
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    if rows is None:
        rp, n_rows = None, n_q
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        rp, n_rows = rows.ctypes.data_as(_i64p), rows.shape[0]
    O = np.empty(lead + (n_rows, d_v)); L = np.empty(lead + (n_rows,))
    _check(lib().oracle_sdpa_rows(qp, kp, vp, bh, n_q, n_kv, d_k, d_v, scale, int(causal), rp, n_rows,
                                  O.ctypes.data_as(_f64p), L.ctypes.data_as(_f64p),
                                  threads or threads_available()), "oracle_sdpa_rows")
    return O, L


def sdpa_rows_window(q, k, v, scale, left, right, rows=None, threads=None):
    """Like sdpa_rows with a local window: row i (key position p = i + n_kv - n_q) sees keys
    p - left <= j <= p + right; a negative bound leaves that side open."""
    lead = q.shape[:-2]
    n_q, d_k = q.shape[-2:]
    n_kv, d_v = v.shape[-2:]
    bh = int(np.prod(lead, dtype=np.int64)) if lead else 1
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    if rows is None:
        rp, n_rows = None, n_q
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        rp, n_rows = rows.ctypes.data_as(_i64p), rows.shape[0]
    O = np.empty(lead + (n_rows, d_v)); L = np.empty(lead + (n_rows,))
    _check(lib().oracle_sdpa_rows_window(qp, kp, vp, bh, n_q, n_kv, d_k, d_v, scale, int(left), int(right), rp,
                                         n_rows, O.ctypes.data_as(_f64p), L.ctypes.data_as(_f64p),
                                         threads or threads_available()), "oracle_sdpa_rows_window")
    return O, L


def decode(q, k, v, lens, scale, pairs=None, threads=None):
    """q [B, H, d_k], k/v [B, H, n_cap, d], lens [B]. Returns O [n_pairs, d_v], LSE [n_pairs]."""
    B, H, n_cap, d_k = k.shape
    d_v = v.shape[-1]
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    if pairs is None:
        pp, n_pairs = None, B * H
    else:
        pairs = np.ascontiguousarray(pairs, dtype=np.int64)
        pp, n_pairs = pairs.ctypes.data_as(_i64p), pairs.shape[0]
    O = np.empty((n_pairs, d_v)); L = np.empty((n_pairs,))
    _check(lib().oracle_decode(qp, kp, vp, lens.ctypes.data_as(_i32p), B, H, n_cap, d_k, d_v, scale, pp,
                               n_pairs, O.ctypes.data_as(_f64p), L.ctypes.data_as(_f64p),
                               threads or threads_available()), "oracle_decode")
    return O, L


def decode_gqa(q, k, v, lens, scale, pairs=None, threads=None):
    """Grouped-query decode. q [B, H_q, d_k], k/v [B, H_kv, n_cap, d], lens [B]; query head h reads
    key/value head h // (H_q // H_kv).  Returns O [n_pairs, d_v], LSE [n_pairs] (pairs = b*H_q + h)."""
    B, H_kv, n_cap, d_k = k.shape
    H_q = q.shape[1]
    d_v = v.shape[-1]
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    lens = np.ascontiguousarray(lens, dtype=np.int32)
    if pairs is None:
        pp, n_pairs = None, B * H_q
    else:
        pairs = np.ascontiguousarray(pairs, dtype=np.int64)
        pp, n_pairs = pairs.ctypes.data_as(_i64p), pairs.shape[0]
    O = np.empty((n_pairs, d_v)); L = np.empty((n_pairs,))
    _check(lib().oracle_decode_gqa(qp, kp, vp, lens.ctypes.data_as(_i32p), B, H_q, H_kv, n_cap, d_k, d_v, scale,
                                   pp, n_pairs, O.ctypes.data_as(_f64p), L.ctypes.data_as(_f64p),
                                   threads or threads_available()), "oracle_decode_gqa")
    return O, L


def sdpa_backward(q, k, v, do, scale, causal=False, q_rows=None, k_rows=None, threads=None):
    """Gradients of exact attention for loss gradient `do`, over leading slice dims.

    q [..., n_q, d_k], k [..., n_kv, d_k], v [..., n_kv, d_v], do [..., n_q, d_v].
    q_rows / k_rows: None (all) or 1-D index arrays applied to every slice.
    Returns dQ [..., n_qr, d_k], dK [..., n_kr, d_k], dV [..., n_kr, d_v] in float64.
    """
    lead = q.shape[:-2]
    n_q, d_k = q.shape[-2:]
    n_kv, d_v = v.shape[-2:]
    bh = int(np.prod(lead, dtype=np.int64)) if lead else 1
    q, qp = _f32(q)
    k, kp = _f32(k)
    v, vp = _f32(v)
    do, dop = _f32(do)
    if q_rows is None:
        qrp, n_qr = None, n_q
    else:
        q_rows = np.ascontiguousarray(q_rows, dtype=np.int64)
        qrp, n_qr = q_rows.ctypes.data_as(_i64p), q_rows.shape[0]
    if k_rows is None:
        krp, n_kr = None, n_kv
    else:
        k_rows = np.ascontiguousarray(k_rows, dtype=np.int64)
        krp, n_kr = k_rows.ctypes.data_as(_i64p), k_rows.shape[0]
    dQ = np.empty(lead + (n_qr, d_k)); dK = np.empty(lead + (n_kr, d_k)); dV = np.empty(lead + (n_kr, d_v))
    _check(lib().oracle_sdpa_backward(qp, kp, vp, dop, bh, n_q, n_kv, d_k, d_v, scale, int(causal), qrp, n_qr, krp,
                                      n_kr, dQ.ctypes.data_as(_f64p), dK.ctypes.data_as(_f64p),
                                      dV.ctypes.data_as(_f64p), threads or threads_available()),
           "oracle_sdpa_backward")
    return dQ, dK, dV
