"""Python binding of libsdpa.so, the B200 exact-attention library (C ABI in include/sdpa.h).

Argument marshalling only: every step of attention runs in the library's CUDA
kernels.  PyTorch is used for device tensors and streams.  There is no CPU
fallback: if libsdpa.so is missing, importing this package fails.

    import memory_optimal_sdpa_b200 as sdpa
    O, LSE = sdpa.fwd(q, k, v, causal=True)                 # bf16, tcgen05 tensor cores
    O, LSE = sdpa.fwd_f32(q, k, v)                          # fp32 on CUDA cores
    O, LSE = sdpa.decode(q, k_cache, v_cache, kv_lens)      # one row per (batch, head)
    O, LSE = sdpa.decode_gqa(q, k_cache, v_cache, kv_lens)  # query heads sharing key/value heads
    dQ, dK, dV = sdpa.bwd(q, k, v, O, dO, LSE, causal=True) # gradients of fwd
"""
import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsdpa.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libsdpa.so is not built: run `python memory_optimal_sdpa_b200/build.py` "
                      "(nvcc, sm_100a).  There is no fallback implementation.")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.sdpa_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
lib.sdpa_fwd.restype = _i
lib.sdpa_fwd_window.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp]
lib.sdpa_fwd_window.restype = _i
lib.sdpa_fwd_f32.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
lib.sdpa_fwd_f32.restype = _i
lib.sdpa_decode_workspace_size.argtypes = [_i, _i, _i, _i]
lib.sdpa_decode_workspace_size.restype = _sz
lib.sdpa_decode.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]
lib.sdpa_decode.restype = _i
lib.sdpa_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _vp]
lib.sdpa_decode_noalloc.restype = _i
lib.sdpa_decode_gqa_workspace_size.argtypes = [_i, _i, _i, _i, _i]
lib.sdpa_decode_gqa_workspace_size.restype = _sz
lib.sdpa_decode_gqa.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _sz, _vp]
lib.sdpa_decode_gqa.restype = _i
lib.sdpa_bwd_workspace_size.argtypes = [_i, _i, _i]
lib.sdpa_bwd_workspace_size.restype = _sz
lib.sdpa_bwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _vp, _sz, _vp]
lib.sdpa_bwd.restype = _i
lib.sdpa_get_last_device_error.argtypes = [_vp]
lib.sdpa_get_last_device_error.restype = _i
lib.sdpa_status_string.argtypes = [_i]
lib.sdpa_status_string.restype = ctypes.c_char_p

SDPA_OK = 0
SDPA_ERR_INVALID_ARG = 1
SDPA_ERR_UNSUPPORTED = 2
SDPA_ERR_MISALIGNED = 3
SDPA_ERR_WORKSPACE = 4
SDPA_ERR_CUDA = 5
SDPA_ERR_DEVICE_TIMEOUT = 6
SDPA_ERR_DEVICE_BAD_LENGTH = 7


class SdpaError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, status_string(status)))


def status_string(status):
    return lib.sdpa_status_string(status).decode()


def _check(status, where):
    if status != SDPA_OK:
        raise SdpaError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _outputs(q, n_q, d_v, dtype, o, lse, want_lse):
    import torch
    B, H = q.shape[0], q.shape[1]
    if o is None:
        o = torch.empty((B, H, n_q, d_v), dtype=dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, device=q.device)
    return o, lse


def fwd(q, k, v, causal=False, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """bf16 prefill. q [B,H,n_q,d], k/v [B,H,n_kv,d] contiguous CUDA bf16; d in {64,128}."""
    B, H, n_q, d_k = q.shape
    n_kv, d_v = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    o, lse = _outputs(q, n_q, d_v, q.dtype, o, lse, want_lse)
    _check(lib.sdpa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k, d_v,
                        float(scale), int(bool(causal)), _stream(stream)), "sdpa_fwd")
    return o, lse


def fwd_window(q, k, v, window_left, window_right, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """bf16 prefill with a local window: row i (key position p = i + n_kv - n_q) sees keys
    p - window_left .. p + window_right; -1 leaves a side open."""
    B, H, n_q, d_k = q.shape
    n_kv, d_v = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    o, lse = _outputs(q, n_q, d_v, q.dtype, o, lse, want_lse)
    _check(lib.sdpa_fwd_window(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k, d_v,
                               float(scale), int(window_left), int(window_right), _stream(stream)), "sdpa_fwd_window")
    return o, lse


def fwd_f32(q, k, v, causal=False, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """fp32 prefill on CUDA cores. Shapes as fwd; d_k, d_v <= 128."""
    B, H, n_q, d_k = q.shape
    n_kv, d_v = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    o, lse = _outputs(q, n_q, d_v, q.dtype, o, lse, want_lse)
    _check(lib.sdpa_fwd_f32(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k, d_v,
                            float(scale), int(bool(causal)), _stream(stream)), "sdpa_fwd_f32")
    return o, lse


def decode_workspace_size(batch, heads, n_kv_cap, d_v):
    return int(lib.sdpa_decode_workspace_size(batch, heads, n_kv_cap, d_v))


def decode(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Decode. q [B,H,d], k/v [B,H,n_cap,d] bf16, kv_lens int32 [B] on the device."""
    import torch
    B, H, n_cap, d_k = k.shape
    d_v = v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    if o is None:
        o = torch.empty((B, H, d_v), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, H, n_cap, d_v)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sdpa_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H, n_cap, d_k, d_v,
                           float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                           _stream(stream)), "sdpa_decode")
    return o, lse


def decode_noalloc(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """Decode without a workspace: for callers that may not allocate device memory.

    Uses the library's fixed device scratch array (see sdpa_decode_noalloc in
    include/sdpa.h).  o and lse are allocated here only when not given.
    """
    import torch
    B, H, n_cap, d_k = k.shape
    d_v = v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    if o is None:
        o = torch.empty((B, H, d_v), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    _check(lib.sdpa_decode_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H, n_cap, d_k,
                                   d_v, float(scale), _stream(stream)), "sdpa_decode_noalloc")
    return o, lse


def decode_gqa_workspace_size(batch, heads_q, heads_kv, n_kv_cap, d_v):
    return int(lib.sdpa_decode_gqa_workspace_size(batch, heads_q, heads_kv, n_kv_cap, d_v))


def decode_gqa(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Grouped-query decode. q [B, H_q, d], k/v [B, H_kv, n_cap, d] bf16 (H_q a multiple of H_kv),
    kv_lens int32 [B] on the device; query head h reads key/value head h // (H_q // H_kv)."""
    import torch
    B, H_kv, n_cap, d_k = k.shape
    H_q = q.shape[1]
    d_v = v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=q.device)
    need = decode_gqa_workspace_size(B, H_q, H_kv, n_cap, d_v)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sdpa_decode_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H_q, H_kv, n_cap,
                               d_k, d_v, float(scale), _ptr(workspace), workspace.numel() * workspace.element_size(),
                               _stream(stream)), "sdpa_decode_gqa")
    return o, lse


def bwd_workspace_size(batch, heads, n_q):
    return int(lib.sdpa_bwd_workspace_size(batch, heads, n_q))


def bwd(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of fwd: returns dQ, dK, dV (bf16, shapes of q, k, v) for loss gradient `do`,
    from the forward's inputs, output `o` and `lse`."""
    import torch
    B, H, n_q, d_k = q.shape
    n_kv, d_v = v.shape[2], v.shape[3]
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    need = bwd_workspace_size(B, H, n_q)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(lib.sdpa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                        n_q, n_kv, d_k, d_v, float(scale), int(bool(causal)), _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _stream(stream)), "sdpa_bwd")
    return dq, dk, dv


def get_last_device_error(stream=None):
    return int(lib.sdpa_get_last_device_error(_stream(stream)))
