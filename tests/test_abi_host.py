"""Host-side checks of the C ABI: runs without a GPU (no compute call reaches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdpa.h")


@pytest.fixture(scope="module")
def sdpa():
    import importlib.util
    spec = importlib.util.spec_from_file_location("_sdpa_build", os.path.join(ROOT, "memory_optimal_sdpa_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import memory_optimal_sdpa_b200 as m
    return m


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdpa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted([
        "sdpa_bwd", "sdpa_bwd_workspace_size", "sdpa_decode", "sdpa_decode_gqa", "sdpa_decode_gqa_workspace_size", "sdpa_decode_noalloc",
        "sdpa_decode_workspace_size", "sdpa_fwd", "sdpa_fwd_f32",
        "sdpa_fwd_window",
        "sdpa_get_last_device_error", "sdpa_status_string"])


def test_library_exports_every_declared_symbol(sdpa):
    lib = ctypes.CDLL(sdpa.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_no_torch_or_oracle_in_the_product_library(sdpa):
    # the shared library links neither torch nor the oracle
    import subprocess
    out = subprocess.run(["ldd", sdpa.LIB_PATH], capture_output=True, text=True).stdout
    assert "torch" not in out and "oracle" not in out
    for f in os.listdir(os.path.join(ROOT, "memory_optimal_sdpa_b200", "csrc")):
        src = open(os.path.join(ROOT, "memory_optimal_sdpa_b200", "csrc", f)).read()
        assert "oracle" not in src.lower().replace("oracle.h", "") or f.endswith(".md"), f


P = 0x10000  # an aligned, never-dereferenced stand-in address


def fwd(sdpa, Q=P, K=P, V=P, O=P, LSE=None, b=1, h=1, nq=128, nkv=128, dk=64, dv=64, scale=0.125, causal=0):
    return sdpa.lib.sdpa_fwd(Q, K, V, O, LSE, b, h, nq, nkv, dk, dv, scale, causal, None)


def test_fwd_argument_errors(sdpa):
    assert fwd(sdpa, Q=None) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, O=None) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, nkv=0) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, b=-1) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, causal=2) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, scale=float("nan")) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, scale=float("inf")) == sdpa.SDPA_ERR_INVALID_ARG
    assert fwd(sdpa, dk=96, dv=96) == sdpa.SDPA_ERR_UNSUPPORTED
    assert fwd(sdpa, dk=64, dv=128) == sdpa.SDPA_ERR_UNSUPPORTED
    # any finite scale passes the argument checks (zero and negative included): the next
    # check to fail is the planted misalignment, not the scale
    assert fwd(sdpa, scale=0.0, O=P + 2) == sdpa.SDPA_ERR_MISALIGNED
    assert fwd(sdpa, scale=-0.5, K=P + 8) == sdpa.SDPA_ERR_MISALIGNED
    assert fwd(sdpa, K=P + 8) == sdpa.SDPA_ERR_MISALIGNED
    assert fwd(sdpa, O=P + 2) == sdpa.SDPA_ERR_MISALIGNED
    assert fwd(sdpa, LSE=P + 2) == sdpa.SDPA_ERR_MISALIGNED
    # degenerate shapes are a successful no-op (no pointer is needed, nothing launches)
    assert fwd(sdpa, Q=None, K=None, V=None, O=None, nq=0) == sdpa.SDPA_OK
    assert fwd(sdpa, Q=None, K=None, V=None, O=None, b=0) == sdpa.SDPA_OK
    assert fwd(sdpa, Q=None, K=None, V=None, O=None, h=0) == sdpa.SDPA_OK


def test_fwd_window_argument_errors(sdpa):
    f = lambda **kw: sdpa.lib.sdpa_fwd_window(*[kw.get(n, d) for n, d in (
        ("Q", P), ("K", P), ("V", P), ("O", P), ("LSE", None), ("b", 1), ("h", 1), ("nq", 64), ("nkv", 64), ("dk", 64),
        ("dv", 64), ("scale", 0.125), ("wl", 16), ("wr", 0), ("st", None))])
    assert f(wl=-2) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(wr=-3) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(Q=None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(dk=96, dv=96) == sdpa.SDPA_ERR_UNSUPPORTED
    assert f(V=P + 2) == sdpa.SDPA_ERR_MISALIGNED
    assert f(V=P + 2, scale=-0.25) == sdpa.SDPA_ERR_MISALIGNED and f(V=P + 2, scale=0.0) == sdpa.SDPA_ERR_MISALIGNED
    assert f(Q=None, K=None, V=None, O=None, nq=0) == sdpa.SDPA_OK


def test_fwd_f32_argument_errors(sdpa):
    f = sdpa.lib.sdpa_fwd_f32
    assert f(None, P, P, P, None, 1, 1, 4, 4, 8, 8, 1.0, 0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(P, P, P, P, None, 1, 1, 4, 4, 0, 8, 1.0, 0, None) == sdpa.SDPA_ERR_INVALID_ARG
    assert f(P, P, P, P, None, 1, 1, 4, 4, 129, 8, 1.0, 0, None) == sdpa.SDPA_ERR_UNSUPPORTED
    assert f(P, P + 2, P, P, None, 1, 1, 4, 4, 8, 8, 1.0, 0, None) == sdpa.SDPA_ERR_MISALIGNED
    assert f(P, P, P, P, None, 1, 1, 0, 4, 8, 8, 1.0, 0, None) == sdpa.SDPA_OK


def test_decode_workspace_and_errors(sdpa):
    ws = sdpa.decode_workspace_size
    assert ws(0, 1, 16, 128) == 0 and ws(1, 1, 0, 128) == 0
    # 64 x 32 heads x 16384-row cache: 512-key splits, 32 per head, each d_v + 1 floats
    assert ws(64, 32, 16384, 128) == 64 * 32 * 32 * 129 * 4
    # a tiny problem uses smaller splits so the grid still fills the GPU
    assert ws(1, 1, 1000, 64) == 16 * 65 * 4
    d = sdpa.lib.sdpa_decode
    need = ws(2, 2, 256, 64)
    args = lambda **kw: dict(dict(Q=P, K=P, V=P, L=P, O=P, LSE=None, b=2, h=2, cap=256, dk=64, dv=64,
                                  scale=0.1, ws=P, wsb=need), **kw)
    call = lambda a: d(a["Q"], a["K"], a["V"], a["L"], a["O"], a["LSE"], a["b"], a["h"], a["cap"], a["dk"], a["dv"],
                       a["scale"], a["ws"], a["wsb"], None)
    assert call(args(ws=None)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(wsb=need - 1)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(L=None)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(cap=0)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(dk=80, dv=80)) == sdpa.SDPA_ERR_UNSUPPORTED
    assert call(args(V=P + 4)) == sdpa.SDPA_ERR_MISALIGNED
    assert call(args(b=0)) == sdpa.SDPA_OK


def test_decode_gqa_workspace_and_errors(sdpa):
    ws = sdpa.decode_gqa_workspace_size
    assert ws(0, 8, 1, 16, 128) == 0 and ws(1, 6, 4, 16, 128) == 0 and ws(1, 8, 0, 16, 128) == 0
    # 64 batches x 64 query heads over 8 key/value heads, 16384-row cache, d = 128 (tensor-core
    # path): 4096-key splits, 4 per head, each d_v + 1 floats per query head
    assert ws(64, 64, 8, 16384, 128) == 64 * 64 * 4 * 129 * 4
    # few (batch, group) pairs: the split halves until the grid has 4 CTAs per SM or reaches 128
    # keys (1 x 8 groups over a 16384-row cache: 128-key splits, 128 per group)
    assert ws(1, 64, 8, 16384, 128) == 1 * 64 * 128 * 129 * 4
    # group size one is plain decode and sizes like it
    assert ws(64, 32, 32, 16384, 128) == sdpa.decode_workspace_size(64, 32, 16384, 128)
    d = sdpa.lib.sdpa_decode_gqa
    need = ws(2, 8, 2, 256, 128)
    args = lambda **kw: dict(dict(Q=P, K=P, V=P, L=P, O=P, LSE=None, b=2, hq=8, hkv=2, cap=256, dk=128, dv=128,
                                  scale=0.1, ws=P, wsb=need), **kw)
    call = lambda a: d(a["Q"], a["K"], a["V"], a["L"], a["O"], a["LSE"], a["b"], a["hq"], a["hkv"], a["cap"],
                       a["dk"], a["dv"], a["scale"], a["ws"], a["wsb"], None)
    assert call(args(ws=None)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(wsb=need - 1)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(hkv=3)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(hkv=0)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(L=None)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(scale=float("nan"))) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(dk=96, dv=96)) == sdpa.SDPA_ERR_UNSUPPORTED
    assert call(args(K=P + 8)) == sdpa.SDPA_ERR_MISALIGNED
    assert call(args(b=0)) == sdpa.SDPA_OK and call(args(hq=0)) == sdpa.SDPA_OK


def test_bwd_workspace_and_errors(sdpa):
    ws = sdpa.bwd_workspace_size
    assert ws(0, 1, 16) == 0 and ws(1, 1, 0) == 0
    # D and LSE log2(e), 64 fp32 dQ accumulator columns and 8 words of per-query terms, per row padded to 128
    assert ws(4, 16, 2048) == 74 * 4 * 16 * 2048 * 4 and ws(1, 2, 130) == 74 * 2 * 256 * 4
    d = sdpa.lib.sdpa_bwd
    need = ws(1, 2, 256)
    args = lambda **kw: dict(dict(Q=P, K=P, V=P, O=P, dO=P, L=P, dQ=P, dK=P, dV=P, b=1, h=2, nq=256, nkv=256, dk=64,
                                  dv=64, scale=0.125, causal=1, ws=P, wsb=need), **kw)
    call = lambda a: d(a["Q"], a["K"], a["V"], a["O"], a["dO"], a["L"], a["dQ"], a["dK"], a["dV"], a["b"], a["h"],
                       a["nq"], a["nkv"], a["dk"], a["dv"], a["scale"], a["causal"], a["ws"], a["wsb"], None)
    assert call(args(ws=None)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(wsb=need - 1)) == sdpa.SDPA_ERR_WORKSPACE
    assert call(args(L=None)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(dO=None)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(nkv=0)) == sdpa.SDPA_ERR_INVALID_ARG
    assert call(args(dk=128, dv=64)) == sdpa.SDPA_ERR_UNSUPPORTED
    assert call(args(scale=-1.0, dQ=P + 2)) == sdpa.SDPA_ERR_MISALIGNED
    assert call(args(scale=0.0, dK=P + 2)) == sdpa.SDPA_ERR_MISALIGNED
    assert call(args(dQ=P + 2)) == sdpa.SDPA_ERR_MISALIGNED
    assert call(args(nq=0)) == sdpa.SDPA_OK


def test_status_strings(sdpa):
    names = ["SDPA_OK", "SDPA_ERR_INVALID_ARG", "SDPA_ERR_UNSUPPORTED", "SDPA_ERR_MISALIGNED", "SDPA_ERR_WORKSPACE",
             "SDPA_ERR_CUDA", "SDPA_ERR_DEVICE_TIMEOUT", "SDPA_ERR_DEVICE_BAD_LENGTH", "SDPA_ERR_DEVICE_CHECK"]
    for code, name in enumerate(names):
        assert sdpa.status_string(code) == name
        assert getattr(sdpa, name) == code
    assert sdpa.status_string(99) == "SDPA_UNKNOWN_STATUS"
    hdr = open(HEADER).read()
    for code, name in enumerate(names):
        assert re.search(r"\b%s\s*=\s*%d\b" % (name, code), hdr), name
