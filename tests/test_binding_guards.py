"""The Python binding's argument guards (CPU: no GPU needed).

The C ABI receives raw pointers and sizes, so a transposed view, a tensor of
another dtype, a shape that disagrees between q, k and v, or a tensor on the
host would reach the kernels as garbage.  The binding rejects each of these
before the library call; these tests check every rejection with host tensors
(the device check runs last, so all others are reachable without a GPU).
"""
import pytest

torch = pytest.importorskip("torch")
sdpa = pytest.importorskip("memory_optimal_sdpa_b200")

bf = torch.bfloat16


def t(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


PREFILL = [sdpa.fwd, sdpa.fwd_f32, lambda q, k, v, **kw: sdpa.fwd_window(q, k, v, 8, 0, **kw)]


def _dtype_for(fn):
    return torch.float32 if fn is sdpa.fwd_f32 else bf


@pytest.mark.parametrize("fn", PREFILL)
def test_prefill_rejects_wrong_dtype(fn):
    dt = _dtype_for(fn)
    other = torch.float16
    with pytest.raises(TypeError, match="q must be"):
        fn(t(1, 2, 8, 64, dtype=other), t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt))
    with pytest.raises(TypeError, match="v must be"):
        fn(t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=other))


@pytest.mark.parametrize("fn", PREFILL)
def test_prefill_rejects_transposed_view(fn):
    dt = _dtype_for(fn)
    q = t(1, 8, 2, 64, dtype=dt).transpose(1, 2)  # a [B, n, H, d] tensor viewed as [B, H, n, d]
    with pytest.raises(ValueError, match="q must be contiguous"):
        fn(q, t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt))


@pytest.mark.parametrize("fn", PREFILL)
def test_prefill_rejects_mismatched_shapes(fn):
    dt = _dtype_for(fn)
    with pytest.raises(ValueError, match="k has shape"):  # heads differ
        fn(t(1, 2, 8, 64, dtype=dt), t(1, 3, 8, 64, dtype=dt), t(1, 3, 8, 64, dtype=dt))
    with pytest.raises(ValueError, match="k has shape"):  # batch differs
        fn(t(2, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt))
    with pytest.raises(ValueError, match="k has shape"):  # head dim differs
        fn(t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 128, dtype=dt), t(1, 2, 8, 64, dtype=dt))
    with pytest.raises(ValueError, match="v has shape"):  # key count differs
        fn(t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt), t(1, 2, 9, 64, dtype=dt))
    with pytest.raises(ValueError, match="q has shape"):  # not 4-D
        fn(t(2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt))


@pytest.mark.parametrize("fn", PREFILL)
def test_prefill_rejects_bad_outputs(fn):
    dt = _dtype_for(fn)
    q, k, v = t(1, 2, 8, 64, dtype=dt), t(1, 2, 16, 64, dtype=dt), t(1, 2, 16, 64, dtype=dt)
    with pytest.raises(ValueError, match="o has shape"):
        fn(q, k, v, o=t(1, 2, 16, 64, dtype=dt))
    with pytest.raises(TypeError, match="lse must be"):
        fn(q, k, v, o=t(1, 2, 8, 64, dtype=dt), lse=t(1, 2, 8, dtype=torch.float64))


@pytest.mark.parametrize("fn", PREFILL)
def test_prefill_rejects_host_tensors(fn):
    dt = _dtype_for(fn)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt), t(1, 2, 8, 64, dtype=dt))


def test_prefill_rejects_non_tensor():
    with pytest.raises(TypeError, match="must be a torch.Tensor"):
        sdpa.fwd([[0.0]], t(1, 2, 8, 64), t(1, 2, 8, 64))


@pytest.mark.parametrize("fn", [sdpa.decode, sdpa.decode_noalloc])
def test_decode_guards(fn):
    q, k, v = t(2, 4, 128), t(2, 4, 64, 128), t(2, 4, 64, 128)
    lens = torch.tensor([64, 3], dtype=torch.int32)
    with pytest.raises(TypeError, match="kv_lens must be"):
        fn(q, k, v, lens.long())
    with pytest.raises(ValueError, match="kv_lens has shape"):
        fn(q, k, v, torch.tensor([64], dtype=torch.int32))
    with pytest.raises(ValueError, match="q has shape"):  # heads of q and the cache differ
        fn(t(2, 8, 128), k, v, lens)
    with pytest.raises(ValueError, match="v has shape"):
        fn(q, k, t(2, 4, 32, 128), lens)
    with pytest.raises(ValueError, match="k must be contiguous"):
        fn(q, t(2, 64, 4, 128).transpose(1, 2), v, lens)
    with pytest.raises(TypeError, match="q must be"):
        fn(q.float(), k, v, lens)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn(q, k, v, lens)


def test_decode_gqa_guards():
    q, k, v = t(2, 8, 128), t(2, 2, 64, 128), t(2, 2, 64, 128)
    lens = torch.tensor([64, 3], dtype=torch.int32)
    with pytest.raises(ValueError, match="q has shape"):  # batch differs
        sdpa.decode_gqa(t(3, 8, 128), k, v, lens)
    with pytest.raises(ValueError, match="o has shape"):
        sdpa.decode_gqa(q, k, v, lens, o=t(2, 2, 128))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        sdpa.decode_gqa(q, k, v, lens)


def test_backward_guards():
    q, k, v = t(1, 2, 8, 64), t(1, 2, 16, 64), t(1, 2, 16, 64)
    o, do, lse = t(1, 2, 8, 64), t(1, 2, 8, 64), t(1, 2, 8, dtype=torch.float32)
    with pytest.raises(ValueError, match="do has shape"):
        sdpa.bwd(q, k, v, o, t(1, 2, 16, 64), lse)
    with pytest.raises(TypeError, match="lse must be"):
        sdpa.bwd(q, k, v, o, do, lse.double())
    with pytest.raises(ValueError, match="o must be contiguous"):
        sdpa.bwd(q, k, v, t(1, 2, 64, 8).transpose(2, 3), do, lse)
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        sdpa.bwd(q, k, v, o, do, lse)
