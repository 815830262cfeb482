"""The five synthetic workloads and their seeded inputs (shapes and value distributions only).

  cfg1  fp32 prefill, B=1 H=1 n_q=n_kv=128 d=64, Q,K,V ~ N(0,1), scale 1/8, non-causal
  cfg2  bf16 prefill, B=4 H=16 n=2048 d=64, Q,K,V ~ N(0,1), scale 1/8, non-causal and causal
  cfg3  bf16 prefill, B=1 H=32 n=8192 d=128, Q,K ~ N(0,1), V ~ U(-1,1), scale 1/sqrt(128), causal
  cfg4  bf16 prefill, B=1 H=8 n=32768 d=128, Q,K ~ N(0, 2.5^2), V ~ N(0,1), scale 1/sqrt(128), non-causal
  cfg5  bf16 decode, B=64 H=32 n_cap=16384 d=128, lengths ~ U{1024..16384}, N(0,1), scale 1/sqrt(128)
  cfg3w cfg3 with a causal local window of 512 keys (window_left = 511, window_right = 0)
  cfg5g cfg5 with grouped-query heads: 64 query heads over 8 key/value heads (groups of 8)

Streams: Q = 0, K = 1, V = 2 (counter = flat element index of the tensor), decode
lengths = 3, sampled rows = 4.  Seed 0 everywhere.  bf16 values are the RNE
rounding of the float32 draw; both the oracle and the GPU consume those bits.
"""
from dataclasses import dataclass, field

import numpy as np

from . import NORMAL, UNIFORM, STREAM_Q, STREAM_K, STREAM_V, bf16_bits_to_f32, fill_host, kv_lengths


@dataclass(frozen=True)
class Dist:
    kind: int = NORMAL
    a: float = 0.0  # mean (normal) or low (uniform)
    b: float = 1.0  # std (normal) or high (uniform)


@dataclass(frozen=True)
class Prefill:
    name: str
    batch: int
    heads: int
    n_q: int
    n_kv: int
    d: int
    causal: bool
    dtype: str  # "bf16" or "f32"
    scale: float
    q: Dist = field(default_factory=Dist)
    k: Dist = field(default_factory=Dist)
    v: Dist = field(default_factory=Dist)
    seed: int = 0
    window: tuple = None  # (left, right) local window, -1 = open side; None = plain causal / full

    @property
    def scale_f32(self):
        return float(np.float32(self.scale))

    def visible_pairs(self):
        """Exact number of (query, key) pairs a window lets through, per (batch, head)."""
        left, right = self.window
        pos = np.arange(self.n_q, dtype=np.int64) + (self.n_kv - self.n_q)
        hi = np.full_like(pos, self.n_kv - 1) if right < 0 else np.minimum(self.n_kv - 1, pos + right)
        lo = np.zeros_like(pos) if left < 0 else np.maximum(0, pos - left)
        return int(np.maximum(0, hi - lo + 1).sum())

    def flops(self):
        """Algorithmic FLOPs: two matmuls at 2 FLOP per multiply-add, halved under a causal mask
        (for a window: 4 d FLOP per visible (query, key) pair)."""
        if self.window is not None:
            return 4.0 * self.d * self.batch * self.heads * self.visible_pairs()
        f = 2.0 * self.batch * self.heads * self.n_q * self.n_kv * (2 * self.d)
        return f / 2 if self.causal else f

    def bytes(self):
        """Algorithmic bytes: Q, K, V read and O, LSE written once."""
        el = 2 if self.dtype == "bf16" else 4
        bh = self.batch * self.heads
        return bh * (self.n_q * self.d * 2 + self.n_kv * self.d * 2) * el + bh * self.n_q * 4

    def with_causal(self, causal):
        return Prefill(**{**self.__dict__, "causal": causal, "name": self.name + ("c" if causal else "")})


@dataclass(frozen=True)
class Decode:
    name: str
    batch: int
    heads: int      # query heads
    n_cap: int
    d: int
    len_lo: int
    len_hi: int
    scale: float
    seed: int = 0
    heads_kv: int = 0  # key/value heads (0: one per query head)

    @property
    def kv_heads(self):
        return self.heads_kv or self.heads

    @property
    def scale_f32(self):
        return float(np.float32(self.scale))

    def lengths(self):
        return kv_lengths(self.batch, self.len_lo, self.len_hi, self.seed)

    def bytes(self, lens=None):
        """Algorithmic bytes: the valid K and V rows, Q, O and LSE (bf16 except LSE)."""
        lens = self.lengths() if lens is None else lens
        kv = int(np.sum(lens, dtype=np.int64)) * self.kv_heads * self.d * 2 * 2
        return kv + self.batch * self.heads * (self.d * 2 * 2 + 4)

    def flops(self, lens=None):
        """Per token n(2 d_K + 2 d_V + 3) (standard attention's decode cost)."""
        lens = self.lengths() if lens is None else lens
        return float(np.sum(lens, dtype=np.int64)) * self.heads * (4 * self.d + 3)


CFG1 = Prefill("cfg1", 1, 1, 128, 128, 64, False, "f32", 1 / 8)
CFG2 = Prefill("cfg2", 4, 16, 2048, 2048, 64, False, "bf16", 1 / 8)
CFG2C = CFG2.with_causal(True)
CFG3 = Prefill("cfg3", 1, 32, 8192, 8192, 128, True, "bf16", 1 / 128 ** 0.5, v=Dist(UNIFORM, -1.0, 1.0))
CFG4 = Prefill("cfg4", 1, 8, 32768, 32768, 128, False, "bf16", 1 / 128 ** 0.5, q=Dist(NORMAL, 0.0, 2.5),
               k=Dist(NORMAL, 0.0, 2.5))
# cfg3's shape with a causal local window of 512 keys (each row sees itself and the 511 before it)
CFG3W = Prefill("cfg3w", 1, 32, 8192, 8192, 128, True, "bf16", 1 / 128 ** 0.5, v=Dist(UNIFORM, -1.0, 1.0),
                window=(511, 0))
CFG5 = Decode("cfg5", 64, 32, 16384, 128, 1024, 16384, 1 / 128 ** 0.5)
# cfg5's batch, cache and lengths with 64 query heads over 8 key/value heads (groups of 8)
CFG5G = Decode("cfg5g", 64, 64, 16384, 128, 1024, 16384, 1 / 128 ** 0.5, heads_kv=8)


def prefill_host(w):
    """Host inputs of a prefill workload: dict of arrays; bf16 as uint16 bits, f32 as float32."""
    bf = w.dtype == "bf16"
    out = {}
    for name, stream, dist, n in (("q", STREAM_Q, w.q, w.n_q), ("k", STREAM_K, w.k, w.n_kv),
                                  ("v", STREAM_V, w.v, w.n_kv)):
        out[name] = fill_host((w.batch, w.heads, n, w.d), w.seed, stream, dist.kind, dist.a, dist.b, bf16=bf)
    return out


def as_f32(x):
    """Exact float32 view of host inputs (bf16 bits widen exactly)."""
    return bf16_bits_to_f32(x) if x.dtype == np.uint16 else x


def to_torch(x, device):
    """Host array (uint16 bf16 bits or float32) -> torch tensor on `device`, same bits."""
    import torch
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(x).to(device)
