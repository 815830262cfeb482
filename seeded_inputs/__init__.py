"""Seeded, counter-based synthetic inputs for tests and benchmarks.

Values are pure functions of (seed, stream, element index): SplitMix64
(Steele, Lea, Flood 2014) for the draws, Box-Muller (1958) for normal
deviates, the top 24 bits for uniform ones, float32 -> bf16 by round to
nearest even.  The host library feeds the oracle; the device library fills
GPU buffers with the same bits.  Nothing here computes attention.

Stream ids used by the workloads: Q = 0, K = 1, V = 2, decode lengths = 3,
sampled query rows = 4.
"""
import ctypes
import os

import numpy as np

from . import build as _build

NORMAL = 0
UNIFORM = 1
STREAM_Q, STREAM_K, STREAM_V, STREAM_LENS, STREAM_ROWS = 0, 1, 2, 3, 4
STREAM_DO = 5  # the loss gradient dO of the backward pass

_host = None
_cuda = None


def _threads():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def host_lib():
    global _host
    if _host is None:
        _build.build(cuda=False)
        lib = ctypes.CDLL(_build.HOST_SO)
        lib.gen_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                 ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_int]
        lib.gen_fill.restype = ctypes.c_int
        lib.gen_draw_u64.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64]
        lib.gen_draw_u64.restype = ctypes.c_uint64
        lib.gen_value_one.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                      ctypes.c_double, ctypes.c_double]
        lib.gen_value_one.restype = ctypes.c_float
        _host = lib
    return _host


def cuda_lib():
    global _cuda
    if _cuda is None:
        if not os.path.exists(_build.CUDA_SO):
            _build.build(cuda=True)
        lib = ctypes.CDLL(_build.CUDA_SO)
        lib.gen_cuda_fill.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint64,
                                      ctypes.c_int, ctypes.c_double, ctypes.c_double, ctypes.c_int,
                                      ctypes.c_void_p, ctypes.c_void_p]
        lib.gen_cuda_fill.restype = ctypes.c_int
        lib.gen_cuda_fill_cache.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_double, ctypes.c_void_p, ctypes.c_void_p]
        lib.gen_cuda_fill_cache.restype = ctypes.c_int
        _cuda = lib
    return _cuda


def fill_host(shape, seed, stream, kind=NORMAL, a=0.0, b=1.0, bf16=True, start=0, threads=None):
    """Elements start.. of a stream as a numpy array of `shape`.

    bf16=True returns uint16 bf16 bit patterns; bf16=False returns float32.
    """
    n = int(np.prod(shape, dtype=np.int64)) if len(shape) else 1
    out = np.empty(shape, dtype=np.uint16 if bf16 else np.float32)
    rc = host_lib().gen_fill(seed, stream, start, n, kind, a, b, 1 if bf16 else 0,
                             out.ctypes.data_as(ctypes.c_void_p), threads or _threads())
    if rc != 0:
        raise ValueError("gen_fill rejected its arguments")
    return out


def bf16_bits_to_f32(bits):
    """Exact widening of bf16 bit patterns to float32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def draw_u64(seed, stream, ctr):
    return int(host_lib().gen_draw_u64(seed, stream, ctr))


def kv_lengths(batch, lo, hi, seed=0):
    """Per-sequence cache lengths, uniform integers in [lo, hi] (inclusive), stream 3."""
    span = hi - lo + 1
    return np.array([lo + ((draw_u64(seed, STREAM_LENS, b) >> 32) * span >> 32) for b in range(batch)],
                    dtype=np.int32)


def sample_rows(n, k, seed=0, salt=0):
    """k distinct row indices in [0, n), always holding 0 and n-1.

    Rows 0 and n-1 are taken first; the other k-2 come from the interior
    [1, n-1) by Floyd's sampling without replacement, drawing from stream 4
    at counters salt*2^32 + i (`salt` separates independent samples, e.g. one
    per head).
    """
    k = min(k, n)
    if k <= 2 or n <= 2:
        return np.array(sorted({0, n - 1})[:max(k, 1)], dtype=np.int64)
    m, want = n - 2, k - 2
    chosen = set()
    ctr = salt << 32
    for j in range(m - want, m):
        t = (draw_u64(seed, STREAM_ROWS, ctr) >> 32) * (j + 1) >> 32
        ctr += 1
        chosen.add(j if t in chosen else t)
    rows = sorted(x + 1 for x in chosen)
    return np.array([0] + rows + [n - 1], dtype=np.int64)


def fill_device(tensor, seed, stream, kind=NORMAL, a=0.0, b=1.0, start=0):
    """Fill a contiguous CUDA tensor (bfloat16 or float32) in place with stream values."""
    import torch
    assert tensor.is_cuda and tensor.is_contiguous()
    if tensor.dtype == torch.bfloat16:
        as_bf16 = 1
    elif tensor.dtype == torch.float32:
        as_bf16 = 0
    else:
        raise TypeError("bf16 or fp32 only")
    rc = cuda_lib().gen_cuda_fill(seed, stream, start, tensor.numel(), kind, a, b, as_bf16,
                                  tensor.data_ptr(), torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError("gen_cuda_fill failed (%d)" % rc)
    return tensor


def fill_device_cache(tensor, lens_dev, seed, stream, kind=NORMAL, a=0.0, b=1.0):
    """Fill a bf16 [B, H, n_cap, d] CUDA cache; rows at or past lens[b] become NaN."""
    import torch
    assert tensor.is_cuda and tensor.is_contiguous() and tensor.dtype == torch.bfloat16
    assert lens_dev.is_cuda and lens_dev.dtype == torch.int32
    B, H, n_cap, d = tensor.shape
    rc = cuda_lib().gen_cuda_fill_cache(seed, stream, B, H, n_cap, d, lens_dev.data_ptr(), kind, a, b,
                                        tensor.data_ptr(), torch.cuda.current_stream().cuda_stream)
    if rc != 0:
        raise RuntimeError("gen_cuda_fill_cache failed (%d)" % rc)
    return tensor
