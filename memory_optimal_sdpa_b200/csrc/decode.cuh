// decode.cuh -- one query row per (batch, head) against a long bf16 KV cache.
//
// Standard attention at decode time reads the whole cache, n(d_K + d_V)
// elements, and does n(2 d_K + 2 d_V + 3) floating-point operations per token
// (blog.hotdry.top SATA article, "scaling bottleneck of standard
// self-attention"): a bandwidth-bound stream, so the kernel is built around
// HBM reads, not arithmetic.
//
// Grouped-query attention (query head h reading key/value head h / group) uses the
// same kernel with a group size above one; the tensor-core kernel in
// decode_gqa.cuh takes the common d = 128 groups.
//
// Split-KV: CTA (split s, head h, batch b) reduces keys [s*chunk, (s+1)*chunk)
// of row b's valid prefix [0, len_b) to a partial (O_s normalised, lse_s).
// Each key is handled by D/8 lanes holding 8 dimensions each (one 16-byte
// read of K and one of V per lane per key, non-allocating in L1); the dot
// product is finished with xor shuffles inside the lane group.  A second
// kernel merges the splits with the same log-sum-exp identity the online
// softmax uses:  lse = M + ln sum_s exp(lse_s - M),
//                O   = sum_s exp(lse_s - lse) O_s.
#pragma once

#include <cuda_bf16.h>

namespace sdpa {

constexpr int DECODE_THREADS = 128;
constexpr int DECODE_UNROLL = 4;  // keys per lane group in flight

// Keys per split for a cache shape: the largest of 512, 256, 128, 64 that still
// yields enough CTAs to fill the GPU (148 SMs x 16).
__host__ __device__ inline int decode_chunk(long long batch, long long heads, long long n_cap) {
  int chunk = 512;
  while (chunk > 64 && batch * heads * ((n_cap + chunk - 1) / chunk) < 148LL * 16) chunk >>= 1;
  return chunk;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* ptr) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr));
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ int decode_len(const int* kv_lens, int b, int n_cap) {
  int len = kv_lens[b];
  if (len < 1 || len > n_cap) {
    record_error(7 /* SDPA_ERR_DEVICE_BAD_LENGTH */);
    len = len < 1 ? 1 : n_cap;
  }
  return len;
}

struct DecodeParams {
  const __nv_bfloat16* Q;  // [B, H, D]
  const __nv_bfloat16* K;  // [B, H_kv, n_cap, D]: query head h reads key/value head h / group
  const __nv_bfloat16* V;
  const int* kv_lens;      // [B]
  float* part_o;           // [B, H, S, D]
  float* part_lse;         // [B, H, S]  (natural log)
  __nv_bfloat16* O;        // [B, H, D]
  float* LSE;              // [B, H] or null
  int H, n_cap, chunk, n_split;
  int H_kv, group;         // H = H_kv * group; group 1 is plain multi-head decode
  float scale_log2;        // scale * log2(e)
};

template <int D>
__global__ void __launch_bounds__(DECODE_THREADS) sdpa_decode_split_kernel(const DecodeParams p) {
  constexpr int LPK = D / 8;             // lanes per key
  constexpr int GPW = 32 / LPK;          // key groups per warp
  constexpr int G = GPW * DECODE_THREADS / 32;  // key groups per CTA
  const int s = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int len = decode_len(p.kv_lens, b, p.n_cap);
  const int k_begin = s * p.chunk;
  if (k_begin >= len) return;
  const int k_end = min(k_begin + p.chunk, len);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = warp * GPW + lane / LPK;  // key group id
  const int e0 = (lane % LPK) * 8;        // first of this lane's 8 dimensions
  const size_t bh = (size_t)b * p.H + h;
  const size_t bkv = (size_t)b * p.H_kv + h / p.group;  // the key/value head this query head reads

  float q[8];
  bf16x8_to_f32(*reinterpret_cast<const uint4*>(p.Q + bh * D + e0), q);
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] *= p.scale_log2;

  const __nv_bfloat16* Kb = p.K + bkv * (size_t)p.n_cap * D + e0;
  const __nv_bfloat16* Vb = p.V + bkv * (size_t)p.n_cap * D + e0;
  const float NEG_INF = -__int_as_float(0x7f800000);
  float m = NEG_INF, l = 0.f, acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  // Trip count is uniform across the CTA so every lane reaches the shuffles.
  for (int base = k_begin; base < k_end; base += G * DECODE_UNROLL) {
    uint4 kr[DECODE_UNROLL], vr[DECODE_UNROLL];
#pragma unroll
    for (int u = 0; u < DECODE_UNROLL; ++u) {
      const int key = base + u * G + g;
      if (key < k_end) {  // rows at or past len are never read
        kr[u] = ld_nc_v4(Kb + (size_t)key * D);
        vr[u] = ld_nc_v4(Vb + (size_t)key * D);
      } else {
        kr[u] = make_uint4(0, 0, 0, 0);
        vr[u] = make_uint4(0, 0, 0, 0);
      }
    }
    float sc[DECODE_UNROLL];
#pragma unroll
    for (int u = 0; u < DECODE_UNROLL; ++u) {
      float kf[8];
      bf16x8_to_f32(kr[u], kf);
      float d = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) d = fmaf(q[i], kf[i], d);
#pragma unroll
      for (int off = LPK / 2; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
      sc[u] = (base + u * G + g < k_end) ? d : NEG_INF;
    }
    float mx = sc[0];
#pragma unroll
    for (int u = 1; u < DECODE_UNROLL; ++u) mx = fmaxf(mx, sc[u]);
    const float m_new = fmaxf(m, mx);
    if (m_new == NEG_INF) continue;
    const float alpha = exp2f(m - m_new);
    l *= alpha;
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] *= alpha;
#pragma unroll
    for (int u = 0; u < DECODE_UNROLL; ++u) {
      const float pu = exp2f(sc[u] - m_new);
      l += pu;
      float vf[8];
      bf16x8_to_f32(vr[u], vf);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = fmaf(pu, vf[i], acc[i]);
    }
    m = m_new;
  }

  // Merge the G lane groups of this CTA.
  __shared__ float s_m[G], s_l[G];
  __shared__ float s_acc[G][D];
  if (lane % LPK == 0) {
    s_m[g] = m;
    s_l[g] = l;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) s_acc[g][e0 + i] = acc[i];
  __syncthreads();
  float M = NEG_INF;
#pragma unroll
  for (int i = 0; i < G; ++i) M = fmaxf(M, s_m[i]);
  float L = 0.f;
  for (int i = 0; i < G; ++i)
    if (s_m[i] != NEG_INF) L += s_l[i] * exp2f(s_m[i] - M);
  const size_t part = bh * p.n_split + s;
  for (int e = threadIdx.x; e < D; e += DECODE_THREADS) {
    float a = 0.f;
    for (int i = 0; i < G; ++i)
      if (s_m[i] != NEG_INF) a += s_acc[i][e] * exp2f(s_m[i] - M);
    p.part_o[part * D + e] = a / L;
  }
  if (threadIdx.x == 0) p.part_lse[part] = M * 0.69314718055994531f + logf(L);
}

template <int D>
__global__ void __launch_bounds__(D) sdpa_decode_combine_kernel(const DecodeParams p) {
  const int bh = blockIdx.x;
  const int b = bh / p.H;
  const int len = decode_len(p.kv_lens, b, p.n_cap);
  const int ns = (len + p.chunk - 1) / p.chunk;
  const float* lse = p.part_lse + (size_t)bh * p.n_split;
  float M = -__int_as_float(0x7f800000);
  for (int s = 0; s < ns; ++s) M = fmaxf(M, lse[s]);
  float L = 0.f, a = 0.f;
  const int e = threadIdx.x;
  const float* po = p.part_o + (size_t)bh * p.n_split * D + e;
  for (int s = 0; s < ns; ++s) {
    const float w = __expf(lse[s] - M);
    L += w;
    a = fmaf(w, po[(size_t)s * D], a);
  }
  p.O[(size_t)bh * D + e] = __float2bfloat16_rn(a / L);
  if (p.LSE && e == 0) p.LSE[bh] = M + logf(L);
}

}  // namespace sdpa
