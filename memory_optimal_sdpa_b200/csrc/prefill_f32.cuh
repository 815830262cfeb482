// prefill_f32.cuh -- exact SDPA forward in fp32 on the CUDA cores.
//
// Same semantics as the bf16 tensor-core kernel (see prefill_bf16.cuh), kept in
// fp32 end to end: scores, softmax weights and the weighted sum of V.  Tensor
// cores are not used because TF32 keeps 10 mantissa bits (~1e-3 relative),
// which cannot meet a 1e-5 relative bound.  Nothing of size n_q x n_kv is
// stored: each warp streams 32-key tiles of K and V through shared memory and
// keeps, per query row, a running maximum, a running sum and the output row.
//
// CTA = 4 warps x 4 query rows; lane i scores key i of the tile against the
// warp's 4 rows, then the weights are broadcast by shuffle and each lane
// accumulates the output dimensions i, i+32, i+64, i+96.
#pragma once

namespace sdpa {

constexpr int F32_ROWS_PER_WARP = 4;
constexpr int F32_WARPS = 4;
constexpr int F32_ROWS = F32_ROWS_PER_WARP * F32_WARPS;  // 16 query rows per CTA
constexpr int F32_KEYS = 32;                             // keys per tile
constexpr int F32_DMAX = 128;

struct F32Params {
  const float* Q;
  const float* K;
  const float* V;
  float* O;
  float* LSE;
  int n_q, n_kv, d_k, d_v;
  float scale;
  int causal;
};

__global__ void __launch_bounds__(128) sdpa_fwd_f32_kernel(const F32Params p) {
  __shared__ float sQ[F32_ROWS][F32_DMAX];
  __shared__ float sK[F32_KEYS][F32_DMAX + 1];  // +1: conflict-free column reads by lane
  __shared__ float sV[F32_KEYS][F32_DMAX];
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * F32_ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int dk = p.d_k, dv = p.d_v;
  const float* Qb = p.Q + (size_t)bh * p.n_q * dk;
  const float* Kb = p.K + (size_t)bh * p.n_kv * dk;
  const float* Vb = p.V + (size_t)bh * p.n_kv * dv;

  for (int i = threadIdx.x; i < F32_ROWS * dk; i += blockDim.x) {
    const int r = i / dk, c = i % dk;
    sQ[r][c] = (r0 + r < p.n_q) ? Qb[(size_t)(r0 + r) * dk + c] : 0.f;
  }

  const float NEG_INF = -__int_as_float(0x7f800000);
  int lim[F32_ROWS_PER_WARP];
  float m[F32_ROWS_PER_WARP], l[F32_ROWS_PER_WARP], acc[F32_ROWS_PER_WARP][4];
  int lim_max = -1;
#pragma unroll
  for (int r = 0; r < F32_ROWS_PER_WARP; ++r) {
    const int row = r0 + warp * F32_ROWS_PER_WARP + r;
    long long c = p.n_kv - 1;
    if (p.causal) {
      const long long cc = (long long)row + p.n_kv - p.n_q;
      if (cc < c) c = cc < -1 ? -1 : cc;
    }
    lim[r] = (row < p.n_q) ? (int)c : -1;
    m[r] = NEG_INF;
    l[r] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[r][e] = 0.f;
  }
  // keys any row of this CTA may see
  {
    const int last = min(r0 + F32_ROWS - 1, p.n_q - 1);
    long long c = p.n_kv - 1;
    if (p.causal) {
      const long long cc = (long long)last + p.n_kv - p.n_q;
      if (cc < c) c = cc;
    }
    lim_max = (int)(c < -1 ? -1 : c);
  }

  for (int k0 = 0; k0 <= lim_max; k0 += F32_KEYS) {
    __syncthreads();
    for (int i = threadIdx.x; i < F32_KEYS * dk; i += blockDim.x) {
      const int r = i / dk, c = i % dk;
      sK[r][c] = (k0 + r < p.n_kv) ? Kb[(size_t)(k0 + r) * dk + c] : 0.f;
    }
    for (int i = threadIdx.x; i < F32_KEYS * dv; i += blockDim.x) {
      const int r = i / dv, c = i % dv;
      sV[r][c] = (k0 + r < p.n_kv) ? Vb[(size_t)(k0 + r) * dv + c] : 0.f;
    }
    __syncthreads();
    float s[F32_ROWS_PER_WARP];
#pragma unroll
    for (int r = 0; r < F32_ROWS_PER_WARP; ++r) s[r] = 0.f;
    for (int c = 0; c < dk; ++c) {
      const float kv = sK[lane][c];
#pragma unroll
      for (int r = 0; r < F32_ROWS_PER_WARP; ++r) s[r] = fmaf(sQ[warp * F32_ROWS_PER_WARP + r][c], kv, s[r]);
    }
#pragma unroll
    for (int r = 0; r < F32_ROWS_PER_WARP; ++r) {
      const float u = (k0 + lane <= lim[r]) ? s[r] * p.scale : NEG_INF;
      float mx = u;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m[r], mx);
      if (m_new == NEG_INF) continue;  // warp-uniform: nothing visible yet for this row
      const float alpha = expf(m[r] - m_new);
      const float pw = expf(u - m_new);
      float sum = pw;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      l[r] = l[r] * alpha + sum;
      m[r] = m_new;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[r][e] *= alpha;
      for (int k = 0; k < F32_KEYS; ++k) {
        const float pk = __shfl_sync(0xffffffffu, pw, k);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = lane + 32 * e;
          if (col < dv) acc[r][e] = fmaf(pk, sV[k][col], acc[r][e]);
        }
      }
    }
  }

#pragma unroll
  for (int r = 0; r < F32_ROWS_PER_WARP; ++r) {
    const int row = r0 + warp * F32_ROWS_PER_WARP + r;
    if (row >= p.n_q) continue;
    const bool any = l[r] > 0.f;
    float* orow = p.O + ((size_t)bh * p.n_q + row) * dv;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = lane + 32 * e;
      if (col < dv) orow[col] = any ? acc[r][e] / l[r] : 0.f;
    }
    if (p.LSE && lane == 0) p.LSE[(size_t)bh * p.n_q + row] = (l[r] > 0.f) ? m[r] + logf(l[r]) : NEG_INF;
  }
}

}  // namespace sdpa
