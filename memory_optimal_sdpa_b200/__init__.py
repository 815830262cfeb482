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
SDPA_ERR_DEVICE_CHECK = 8


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


# ------------------------------------------------------------------------------ argument guards
# The C ABI sees raw pointers and sizes only, so it cannot tell a transposed view, a tensor of
# another dtype or a tensor on another device from a valid argument.  These guards reject such
# tensors before the call.  Order: type, dtype, shape, contiguity, then device (so everything
# but the device check can be exercised with host tensors).
def _tensor(t, name, dtype, shape):
    """t must be a torch tensor of `dtype` whose shape matches `shape` (None entries are free)."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor, got %s" % (name, type(t).__name__))
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != len(shape) or any(want is not None and got != want for got, want in zip(t.shape, shape)):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape),
                                                           tuple("*" if x is None else x for x in shape)))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous (row-major); got strides %s -- pass .contiguous()"
                         % (name, tuple(t.stride())))
    return t


def _device(ref_name, ref, *others):
    """ref must be a CUDA tensor and every other (name, tensor) must live on the same device."""
    if ref.device.type != "cuda":
        raise ValueError("%s must be a CUDA tensor, got device %s" % (ref_name, ref.device))
    for name, t in others:
        if t is not None and t.device != ref.device:
            raise ValueError("%s is on %s but %s is on %s" % (name, t.device, ref_name, ref.device))
    return ref.device


def _stream(stream, device):
    import torch
    s = torch.cuda.current_stream(device) if stream is None else stream
    if s.device != device:
        raise ValueError("stream is on %s but the tensors are on %s" % (s.device, device))
    return ctypes.c_void_p(s.cuda_stream)


def _call(device, fn, *args):
    """Run a library call with `device` current (the C ABI works on the current device)."""
    import torch
    with torch.cuda.device(device):
        return fn(*args)


def _nbytes(t):
    return t.numel() * t.element_size()


def _prefill_args(q, k, v, o, lse, dtype, want_lse):
    """Shapes of a prefill call: q [B,H,n_q,d_k], k [B,H,n_kv,d_k], v [B,H,n_kv,d_v]."""
    import torch
    _tensor(q, "q", dtype, (None, None, None, None))
    B, H, n_q, d_k = q.shape
    _tensor(k, "k", dtype, (B, H, None, d_k))
    n_kv = k.shape[2]
    _tensor(v, "v", dtype, (B, H, n_kv, None))
    d_v = v.shape[3]
    if o is not None:
        _tensor(o, "o", dtype, (B, H, n_q, d_v))
    if lse is not None:
        _tensor(lse, "lse", torch.float32, (B, H, n_q))
    dev = _device("q", q, ("k", k), ("v", v), ("o", o), ("lse", lse))
    if o is None:
        o = torch.empty((B, H, n_q, d_v), dtype=dtype, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, device=dev)
    return B, H, n_q, n_kv, d_k, d_v, o, lse, dev


def fwd(q, k, v, causal=False, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """bf16 prefill. q [B,H,n_q,d], k/v [B,H,n_kv,d] contiguous CUDA bf16; d in {64,128}."""
    import torch
    B, H, n_q, n_kv, d_k, d_v, o, lse, dev = _prefill_args(q, k, v, o, lse, torch.bfloat16, want_lse)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    _check(_call(dev, lib.sdpa_fwd, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k, d_v,
                 float(scale), int(bool(causal)), _stream(stream, dev)), "sdpa_fwd")
    return o, lse


def fwd_window(q, k, v, window_left, window_right, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """bf16 prefill with a local window: row i (key position p = i + n_kv - n_q) sees keys
    p - window_left .. p + window_right; -1 leaves a side open."""
    import torch
    B, H, n_q, n_kv, d_k, d_v, o, lse, dev = _prefill_args(q, k, v, o, lse, torch.bfloat16, want_lse)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    _check(_call(dev, lib.sdpa_fwd_window, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k,
                 d_v, float(scale), int(window_left), int(window_right), _stream(stream, dev)), "sdpa_fwd_window")
    return o, lse


def fwd_f32(q, k, v, causal=False, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """fp32 prefill on CUDA cores. Shapes as fwd; d_k, d_v <= 128."""
    import torch
    B, H, n_q, n_kv, d_k, d_v, o, lse, dev = _prefill_args(q, k, v, o, lse, torch.float32, want_lse)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    _check(_call(dev, lib.sdpa_fwd_f32, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, n_q, n_kv, d_k, d_v,
                 float(scale), int(bool(causal)), _stream(stream, dev)), "sdpa_fwd_f32")
    return o, lse
def _decode_args(q, k, v, kv_lens, o, lse, want_lse, grouped):
    """Shapes of a decode call: q [B,H_q,d_k], k [B,H_kv,n_cap,d_k], v [B,H_kv,n_cap,d_v], kv_lens [B]."""
    import torch
    _tensor(k, "k", torch.bfloat16, (None, None, None, None))
    B, H_kv, n_cap, d_k = k.shape
    _tensor(v, "v", torch.bfloat16, (B, H_kv, n_cap, None))
    d_v = v.shape[3]
    _tensor(q, "q", torch.bfloat16, (B, None if grouped else H_kv, d_k))
    H_q = q.shape[1]
    _tensor(kv_lens, "kv_lens", torch.int32, (B,))
    if o is not None:
        _tensor(o, "o", torch.bfloat16, (B, H_q, d_v))
    if lse is not None:
        _tensor(lse, "lse", torch.float32, (B, H_q))
    dev = _device("q", q, ("k", k), ("v", v), ("kv_lens", kv_lens), ("o", o), ("lse", lse))
    if o is None:
        o = torch.empty((B, H_q, d_v), dtype=torch.bfloat16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, H_q), dtype=torch.float32, device=dev)
    return B, H_q, H_kv, n_cap, d_k, d_v, o, lse, dev


def _workspace(workspace, need, dev):
    import torch
    if workspace is None:
        return torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    if not isinstance(workspace, torch.Tensor) or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous torch.Tensor")
    _device("workspace", workspace)
    if workspace.device != dev:
        raise ValueError("workspace is on %s but the tensors are on %s" % (workspace.device, dev))
    return workspace


def decode_workspace_size(batch, heads, n_kv_cap, d_v):
    return int(lib.sdpa_decode_workspace_size(batch, heads, n_kv_cap, d_v))


def decode(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Decode. q [B,H,d], k/v [B,H,n_cap,d] bf16, kv_lens int32 [B] on the device."""
    B, H, _, n_cap, d_k, d_v, o, lse, dev = _decode_args(q, k, v, kv_lens, o, lse, want_lse, grouped=False)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    workspace = _workspace(workspace, decode_workspace_size(B, H, n_cap, d_v), dev)
    _check(_call(dev, lib.sdpa_decode, _ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H, n_cap,
                 d_k, d_v, float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream, dev)), "sdpa_decode")
    return o, lse


def decode_noalloc(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, stream=None):
    """Decode without a workspace: for callers that may not allocate device memory.

    Uses the library's fixed device scratch array (see sdpa_decode_noalloc in
    include/sdpa.h).  o and lse are allocated here only when not given.
    """
    B, H, _, n_cap, d_k, d_v, o, lse, dev = _decode_args(q, k, v, kv_lens, o, lse, want_lse, grouped=False)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    _check(_call(dev, lib.sdpa_decode_noalloc, _ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H,
                 n_cap, d_k, d_v, float(scale), _stream(stream, dev)), "sdpa_decode_noalloc")
    return o, lse


def decode_gqa_workspace_size(batch, heads_q, heads_kv, n_kv_cap, d_v):
    return int(lib.sdpa_decode_gqa_workspace_size(batch, heads_q, heads_kv, n_kv_cap, d_v))


def decode_gqa(q, k, v, kv_lens, scale=None, o=None, lse=None, want_lse=True, workspace=None, stream=None):
    """Grouped-query decode. q [B, H_q, d], k/v [B, H_kv, n_cap, d] bf16 (H_q a multiple of H_kv),
    kv_lens int32 [B] on the device; query head h reads key/value head h // (H_q // H_kv)."""
    B, H_q, H_kv, n_cap, d_k, d_v, o, lse, dev = _decode_args(q, k, v, kv_lens, o, lse, want_lse, grouped=True)
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    workspace = _workspace(workspace, decode_gqa_workspace_size(B, H_q, H_kv, n_cap, d_v), dev)
    _check(_call(dev, lib.sdpa_decode_gqa, _ptr(q), _ptr(k), _ptr(v), _ptr(kv_lens), _ptr(o), _ptr(lse), B, H_q,
                 H_kv, n_cap, d_k, d_v, float(scale), _ptr(workspace), _nbytes(workspace), _stream(stream, dev)),
           "sdpa_decode_gqa")
    return o, lse


def bwd_workspace_size(batch, heads, n_q):
    return int(lib.sdpa_bwd_workspace_size(batch, heads, n_q))


def bwd(q, k, v, o, do, lse, causal=False, scale=None, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """Gradients of fwd: returns dQ, dK, dV (bf16, shapes of q, k, v) for loss gradient `do`,
    from the forward's inputs, output `o` and `lse`."""
    import torch
    bf = torch.bfloat16
    _tensor(q, "q", bf, (None, None, None, None))
    B, H, n_q, d_k = q.shape
    _tensor(k, "k", bf, (B, H, None, d_k))
    n_kv = k.shape[2]
    _tensor(v, "v", bf, (B, H, n_kv, None))
    d_v = v.shape[3]
    _tensor(o, "o", bf, (B, H, n_q, d_v))
    _tensor(do, "do", bf, (B, H, n_q, d_v))
    _tensor(lse, "lse", torch.float32, (B, H, n_q))
    for name, g, like in (("dq", dq, q), ("dk", dk, k), ("dv", dv, v)):
        if g is not None:
            _tensor(g, name, bf, tuple(like.shape))
    dev = _device("q", q, ("k", k), ("v", v), ("o", o), ("do", do), ("lse", lse), ("dq", dq), ("dk", dk),
                  ("dv", dv))
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    scale = 1.0 / math.sqrt(d_k) if scale is None else scale
    workspace = _workspace(workspace, bwd_workspace_size(B, H, n_q), dev)
    _check(_call(dev, lib.sdpa_bwd, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(do), _ptr(lse), _ptr(dq), _ptr(dk),
                 _ptr(dv), B, H, n_q, n_kv, d_k, d_v, float(scale), int(bool(causal)), _ptr(workspace),
                 _nbytes(workspace), _stream(stream, dev)), "sdpa_bwd")
    return dq, dk, dv


def get_last_device_error(stream=None):
    """Synchronise `stream` (default: the current stream of the current device), then read and
    clear the current device's error word."""
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(lib.sdpa_get_last_device_error(ctypes.c_void_p(s.cuda_stream)))
