// backward.cuh -- gradients of exact SDPA (dQ, dK, dV), bf16 in and out, on the sm_100a tensor cores.
//
// The MoA roadmap ends with the backward pass in the same memory-optimal form
// (agents-report.net MoA article, "implementation roadmap").  Given the saved
// log-sum-exp of every query row, the probabilities are recomputed tile by tile
// and nothing of size n_q x n_kv reaches memory:
//   P  = exp(S scale - LSE)            S = Q K^T
//   dP = dO V^T,   D_i = dO_i . O_i    (= sum_k P_ik dP_ik)
//   dS = P (dP - D)
//   dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K
// Three kernels:
//   pre   D_i and LSE in log2 units (+inf where a row must get P = 0) into a workspace
//   dkdv  one CTA per 128-key tile, streaming the query tiles that see it:
//         S^T = K Q^T and dP^T = V dO^T (tcgen05, fp32 in TMEM), the elementwise
//         P^T and dS^T (bf16, written back over S^T and dP^T), then dV += P^T dO and
//         dK += dS^T Q with the TMEM operand form; dV and dK stay in TMEM to the end
//   d = 64 (fused dQ): dkdv also writes dS^T into shared memory, forms dQ_t = dS_t K for each
//         query tile t it visits (tcgen05, dS read as an MN-major operand, fp32 in TMEM) and
//         reduce-adds it into an fp32 accumulator with a TMA reduce; then
//   dq_out dQ = scale * accumulator in bf16.
//         (At d = 64 with scale != 0 the host runs the one-kernel form of backward_d64.cuh
//         instead; this fused path serves scale 0.)
//   d = 128: dkdv's four accumulators fill TMEM, so dQ has its own kernel:
//   dq    one CTA per 128-row query tile, streaming key tiles: S, dP, dS as above,
//         then dQ += dS K; launched as a programmatic dependent of dkdv (which it does not
//         read), so its CTAs fill the SMs dkdv's tail leaves
// dK and dV are written once; dQ is written once at d = 128 (the price: S and dP formed in
// both kernels) and accumulated in fp32 over the key tiles at d = 64 (S and dP formed once;
// measured 425 -> 557 TF/s on 4 x 16 x 2048, 336 -> 420 causal).  Global traffic stays O(n d).
//
// Warp roles (384 threads, as the forward kernel): warps 0-7 two elementwise
// warpgroups (warpgroup w takes columns [64 w, 64 w + 64) of the 128 x 128
// tile; thread = TMEM lane = the tile's key (dkdv) or query row (dq)), warp 8
// the TMA producer, warp 9 the MMA issuer and TMEM owner (at d = 128 only the
// S / dP one, with warp 10 issuing the gradient products), the rest idle.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

// At d = 128, two MMA issuers: one for the S / dP products, one for the gradient products
// (which also releases the ring stages), so neither waits behind the other's instruction
// stream (measured: d = 128 causal 536 -> 546 TF/s; at d = 64 one issuer is faster, 400 vs 380).
#ifndef SDPA_BWD_TWO_ISSUERS_MIN_D
#define SDPA_BWD_TWO_ISSUERS_MIN_D 128
#endif

#ifndef SDPA_BWD_DS_SEPARATE_D64
#define SDPA_BWD_DS_SEPARATE_D64 0  // measured: d = 64 backward 427 -> 414 TF/s with it, d = 128 709 -> 716
#endif

// d = 64: dQ is formed in the dK/dV kernel (dQ_t = dS_t K for each query tile t it visits, from dS
// in shared memory) and reduce-added in fp32 into a workspace by TMA, so S and dP are computed
// once instead of once per kernel; a small kernel then writes dQ in bf16.  At d = 128 the four
// accumulators of the dK/dV kernel fill TMEM and leave no columns for dQ, so dQ keeps its own kernel.
#ifndef SDPA_BWD_FUSED_DQ_D64
#define SDPA_BWD_FUSED_DQ_D64 1
#endif

// d = 128 dK/dV kernel: the per-query terms -LSE log2(e) / c2 and -D enter the S^T and dP^T products
// as one more K = 16 step against a block of ones (as in the d = 64 kernel), so the elementwise
// step reads no per-column vectors; used when the host supplies the term images (scale != 0).
#ifndef SDPA_BWD_AUG_D128
#define SDPA_BWD_AUG_D128 1
#endif

namespace sdpa {

struct BwdParams {
  const __nv_bfloat16* O;   // [bh, n_q, D]   (pre)
  const __nv_bfloat16* dO;  // [bh, n_q, D]   (pre)
  const float* LSE;         // [bh, n_q], natural log of the scaled logits (pre)
  float* Dvec;              // [bh, n_q_pad]  rowsum(dO * O); 0 in the padding
  float* L2;                // [bh, n_q_pad]  LSE * log2(e); +inf in the padding and for rows without keys
  __nv_bfloat16* dQ;        // [bh, n_q, D]
  __nv_bfloat16* dK;        // [bh, n_kv, D]
  __nv_bfloat16* dV;        // [bh, n_kv, D]
  float* dQacc;             // [bh, n_q_pad, D] fp32 dQ / scale, reduce-added by the dK/dV kernel (fused dQ)
  // d = 64 kernel: per 128-row query tile, four 1 KB shared-memory images (8 rows x 64 queries bf16,
  // 128-byte swizzle): -LSE log2(e) / (scale log2(e)) and -D of each half as three bf16 terms
  uint8_t* aug;
  int n_q, n_kv, n_q_pad, bh_count;
  float scale, scale_log2;
};

template <int D>
struct BwdCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int BLOCK_BYTES = 128 * 64 * 2;
  // fused dQ (d = 64 only, see SDPA_BWD_FUSED_DQ_D64)
  static constexpr bool FUSED_DQ = (D == 64) && SDPA_BWD_FUSED_DQ_D64;
  // d = 64: four stages (three beside the fused dQ's buffers), which also keeps the CTA's shared
  // memory above half an SM's, so a second CTA (that would wait for TMEM) is never placed beside it.
  static constexpr int NSTAGE = (D == 64) ? (FUSED_DQ ? 3 : 4) : 2;
  static constexpr bool AUG = (D == 128) && SDPA_BWD_AUG_D128;
  // dkdv, per query tile after Q and dO: L2[128] then D[128], or (AUG) the four 1 KB images of the
  // per-query terms ([S, dP] x [half])
  static constexpr int VEC_BYTES = AUG ? 4096 : 1024;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + VEC_BYTES;
  static constexpr int FIX_OFF = 0;                // the CTA's fixed pair: (K, V) or (Q, dO)
  static constexpr int ST_OFF = 2 * TILE_BYTES;    // streamed stages: (Q, dO, vectors) or (K, V)
  // fused dQ: two buffers of dS^T (query tile t in buffer t % 2; bf16, 128 keys x 128 queries in
  // two 64-query blocks, 128-byte swizzle), then the fp32 staging of dQ for the reduce (128 rows x
  // 32 columns per elementwise warpgroup, 128-byte swizzle).  Warpgroup 0 stages in the fixed V
  // tile's place: V is read once, into TMEM, before the first S product.
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int DS_OFF = ST_OFF + NSTAGE * STAGE_BYTES;
  static constexpr int STG_OFF = DS_OFF + (FUSED_DQ ? 2 * DS_BYTES : 0);
  static constexpr int STG_BYTES = 128 * 32 * 4;
  // AUG: the ones block (two 64-key images, rows 0-2 = 1) and 2 KB of zeros
  static constexpr int ONES_OFF = STG_OFF + (FUSED_DQ ? STG_BYTES : 0);
  static constexpr int ZERO_OFF = ONES_OFF + (AUG ? 2048 : 0);
  static constexpr int BAR_OFF = ZERO_OFF + (AUG ? 2048 : 0);
  // fix_full, full[NSTAGE], empty[NSTAGE], s_full[2], p_full[2], grad_done[2], o_full, drain[2], fix_tmem,
  // sd_free[2], dq_full, dq_free, ds_free[2], const_ready
  static constexpr int NBAR = 1 + 2 * NSTAGE + 12 + 5;
  static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 16 + 1024;
  static constexpr int THREADS = 384;
  static constexpr int EW_REGS = 192;  // 192 x 256 + 120 x 128 = 168 x 384: no spills in the control warps
  static constexpr int CONTROL_REGS = 120;
  static constexpr int LOAD_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr uint32_t COL_S = 0;      // S or S^T, fp32; then P^T (bf16 pairs) over its first columns
  static constexpr uint32_t COL_DP = 128;   // dP or dP^T, fp32; then dS / dS^T (bf16 pairs)
  static constexpr uint32_t COL_A = 256;    // accumulator: dV (dkdv) or dQ (dq)
  static constexpr uint32_t COL_B = 256 + D;  // accumulator: dK (dkdv)
  static constexpr uint32_t TMEM_COLS = 512;
  static constexpr bool TWO_ISSUERS = D >= SDPA_BWD_TWO_ISSUERS_MIN_D;
  // d = 64: the CTA's fixed pair (K, V in dkdv; Q, dO in dq), the A operands of the S and dP
  // products, is copied once into TMEM columns [384, 448), so those products read only their B
  // operand from shared memory (with both operands there, an N = 64 product moves 6 KB of shared
  // memory per 32 clocks of math, about the SM's shared-memory bandwidth).  At d = 128 the S, dP
  // and gradient accumulators fill all 512 columns.
  static constexpr bool FIX_IN_TMEM = (D == 64);
  static constexpr uint32_t COL_FIX = 384;
  // dq kernel: dS in columns of its own (bf16 pairs, 32 per warpgroup) instead of over dP, so
  // the next key tile's S and dP products need only wait until the elementwise warps have read
  // S and dP, not until the dQ product has read dS.
  static constexpr bool DS_SEPARATE = SDPA_BWD_DS_SEPARATE_D64 || D == 128;
  static constexpr uint32_t COL_DS = FIX_IN_TMEM ? 448 : 384;
  static constexpr uint32_t COL_DQ = 448;  // fused dQ: dQ_t (fp32, D columns) in the dK/dV kernel
  static_assert(!FUSED_DQ || (FIX_IN_TMEM && !TWO_ISSUERS && COL_DQ + D <= TMEM_COLS && TILE_BYTES == STG_BYTES),
                "fused dQ layout");
  static_assert(DS_OFF % 1024 == 0 && STG_OFF % 1024 == 0 && ONES_OFF % 1024 == 0 && ZERO_OFF % 1024 == 0 &&
                    STAGE_BYTES % 1024 == 0,
                "swizzled buffers need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Programmatic dependent launch.  launch_dependents: the next kernel on the stream, if launched
// with programmatic stream serialization, may start once every CTA of this grid has executed it
// (or exited).  wait: block until the grids this one depends on have completed and their memory
// operations are visible (returns at once when there are none).
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// TMEM column of the bf16 pairs holding tile columns [16 kk, 16 kk + 16): warpgroup w packs
// its 64 columns into [64 w, 64 w + 32) of the fp32 region it read them from.
__device__ __forceinline__ uint32_t bwd_pair_col(int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); }

// v as hi + mid + lo, three bf16 values (round to nearest at each step; the remainders are exact
// in fp32, so the sum carries v to 24 bits).  Infinite v: hi = v, mid = lo = 0.
__device__ __forceinline__ void bwd_split3(float v, uint16_t (&t)[3]) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  t[0] = __bfloat16_as_ushort(hi);
  if (!isfinite(v)) {
    t[1] = t[2] = 0;
    return;
  }
  const float r1 = v - __bfloat162float(hi);
  const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(mid);
  t[1] = __bfloat16_as_ushort(mid);
  t[2] = __bfloat16_as_ushort(__float2bfloat16_rn(r2));
}

// ------------------------------------------------------------------------------------ pre
template <int D>
__global__ void __launch_bounds__(128) sdpa_bwd_pre_kernel(const BwdParams p) {
  constexpr int LPR = D / 8;      // lanes per row, 8 elements each
  constexpr int RPW = 32 / LPR;   // rows per warp pass
  const int bh = blockIdx.y;
  const int r0 = blockIdx.x * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e0 = (lane % LPR) * 8;
  const float POS_INF = __int_as_float(0x7f800000);
  if (D == 64 && p.dQacc) {  // the fp32 dQ accumulator of these 128 rows starts at zero
    float4* z = reinterpret_cast<float4*>(p.dQacc + ((size_t)bh * p.n_q_pad + r0) * D);
#pragma unroll 4
    for (int i = threadIdx.x; i < 128 * D / 4; i += 128) z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int it = 0; it < 128 / (4 * RPW); ++it) {
    const int row = r0 + (it * 4 + warp) * RPW + lane / LPR;
    float dot = 0.f;
    if (row < p.n_q) {
      const size_t off = ((size_t)bh * p.n_q + row) * D + e0;
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(p.O + off));
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(p.dO + off));
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        dot = fmaf(__uint_as_float(wa[i] << 16), __uint_as_float(wb[i] << 16), dot);
        dot = fmaf(__uint_as_float(wa[i] & 0xFFFF0000u), __uint_as_float(wb[i] & 0xFFFF0000u), dot);
      }
    }
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (lane % LPR == 0) {
      const size_t o = (size_t)bh * p.n_q_pad + row;
      if (row < p.n_q) {
        const float lse = p.LSE[(size_t)bh * p.n_q + row];
        p.Dvec[o] = dot;
        p.L2[o] = (lse == -POS_INF) ? POS_INF : lse * 1.4426950408889634f;  // no key: P = 0 everywhere
      } else {
        p.Dvec[o] = 0.f;
        p.L2[o] = POS_INF;
      }
    }
  }
  if (p.aug) {
    // The d = 64 kernel and the d = 128 dK/dV kernel add -LSE log2(e) / c2 to S and -D to dP inside the tensor-core products:
    // each value as three bf16 terms (hi + mid + lo holds 24 bits) in rows 0-2 of a 64-query
    // block, rows 3-7 zero, laid out as the kernel's shared memory expects.
    __syncthreads();  // this block's D and LSE log2(e) values are written
    const size_t o = (size_t)bh * p.n_q_pad + r0 + threadIdx.x;
    const float vs = -p.L2[o] / p.scale_log2, vp = -p.Dvec[o];
    uint16_t ts[3], tp[3];
    bwd_split3(vs, ts);
    bwd_split3(vp, tp);
    const int h = threadIdx.x >> 6, col = threadIdx.x & 63;
    uint16_t* img = reinterpret_cast<uint16_t*>(p.aug + ((size_t)bh * (p.n_q_pad / 128) + blockIdx.x) * 4096);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int e = (k * 128 + ((((col * 2) >> 4) ^ k) << 4) + ((col * 2) & 15)) >> 1;  // element within a 1 KB image
      img[h * 512 + e] = k < 3 ? ts[k] : (uint16_t)0;
      img[(2 + h) * 512 + e] = k < 3 ? tp[k] : (uint16_t)0;
    }
  }
}

// ------------------------------------------------------------------------------------ dQ out
// Fused dQ: dQ = scale * dQacc in bf16, rows below n_q (eight elements per thread and pass).
template <int D>
__global__ void __launch_bounds__(256) sdpa_bwd_dq_out_kernel(const BwdParams p) {
  const size_t n8 = (size_t)p.bh_count * p.n_q * (D / 8);
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (size_t)gridDim.x * 256) {
    const size_t row = i / (D / 8);  // bh * n_q + r
    const int c = (int)(i % (D / 8)) * 8;
    const size_t bh = row / p.n_q, r = row % p.n_q;
    const float4* src = reinterpret_cast<const float4*>(p.dQacc + (bh * p.n_q_pad + r) * D + c);
    const float4 a = src[0], b = src[1];
    const float k = p.scale;
    *reinterpret_cast<uint4*>(p.dQ + row * D + c) =
        make_uint4(sm100::pack_bf16x2(a.x * k, a.y * k), sm100::pack_bf16x2(a.z * k, a.w * k),
                   sm100::pack_bf16x2(b.x * k, b.y * k), sm100::pack_bf16x2(b.z * k, b.w * k));
  }
}

// Elementwise step shared by both kernels, for 32 tile columns starting at `c0` of this
// warpgroup's half: P = 2^(S c2 - l2), dS = P (dP - dd), with `keep(c)` false for masked
// entries.  s and dp hold the 32 fp32 values; pp and ps receive the bf16 pairs.
template <class L2F, class DDF, class KEEP>
__device__ __forceinline__ void bwd_elementwise(const uint32_t (&s)[32], const uint32_t (&dp)[32], float c2,
                                                L2F l2, DDF dd, KEEP keep, uint32_t (&pp)[16],
                                                uint32_t (&ps)[16]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float pr[2], dr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = 2 * i + h;
      float e = sm100::ex2_approx(__uint_as_float(s[c]) * c2 - l2(c));
      if (!keep(c)) e = 0.f;
      pr[h] = e;
      dr[h] = e * (__uint_as_float(dp[c]) - dd(c));
    }
    pp[i] = sm100::pack_bf16x2(pr[0], pr[1]);
    ps[i] = sm100::pack_bf16x2(dr[0], dr[1]);
  }
}

// ------------------------------------------------------------------------------------ dK, dV
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    sdpa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                         const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
  using C = BwdCfg<D>;
  using namespace sm100;
  // The dQ kernel after this one on the stream reads nothing it writes: once every CTA of this
  // grid has started, its CTAs may take the SMs this grid's tail leaves.
  griddep_launch_dependents();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sFix = smem + C::FIX_OFF;  // K, V
  uint8_t* sSt = smem + C::ST_OFF;    // per stage: Q, dO, L2[128], D[128]
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* fix_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + C::NSTAGE;
  uint64_t* s_full = empty + C::NSTAGE;  // [half]
  uint64_t* p_full = s_full + 2;         // [half] = [warpgroup]
  uint64_t* grad_done = p_full + 2;      // [half]: the gradient products reading half h completed
  uint64_t* o_full = grad_done + 2;
  uint64_t* drain = o_full + 1;          // [issuer]
  uint64_t* fix_tmem = drain + 2;        // d = 64: the fixed pair has been copied into TMEM
  uint64_t* sd_free = fix_tmem + 1;      // [half] (dq): S and dP of half h are in registers
  uint64_t* dq_full = sd_free + 2;       // fused dQ: dQ_t is in TMEM
  uint64_t* dq_free = dq_full + 1;       // fused dQ: the elementwise warps have read dQ_t
  uint64_t* ds_free = dq_free + 1;       // [buffer] fused dQ: the dQ_t product has read dS buffer t % 2
  uint64_t* const_ready = ds_free + 2;   // AUG: the ones and zero blocks are written
  // AUG at run time: the host supplied the per-query term images (it does when scale != 0)
  const bool aug = C::AUG && p.aug != nullptr;
  uint8_t* sDS = smem + C::DS_OFF;
  uint8_t* sStg[2] = {sFix + C::TILE_BYTES, smem + C::STG_OFF};  // [warpgroup]
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x % p.bh_count;
  const int j0 = (int)(blockIdx.x / p.bh_count) * 128;  // key tile (causal: the first ones see the most rows)
  const int off = p.n_kv - p.n_q;                        // bottom-right alignment
  // Query tiles that see some key of [j0, j0 + 128): causal rows q with q + off >= j0.
  int t_first = 0;
  if (CAUSAL) {
    const long long q_min = (long long)j0 - off;
    t_first = q_min <= 0 ? 0 : (int)(q_min / 128);
  }
  const int n_qt = (p.n_q + 127) / 128;
  const int NT = t_first < n_qt ? n_qt - t_first : 0;

  if (threadIdx.x == 0) {
    mbar_init(fix_full, 1);
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(&grad_done[0], 1);
    mbar_init(&grad_done[1], 1);
    mbar_init(o_full, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(fix_tmem, 256);
    mbar_init(&sd_free[0], 128);
    mbar_init(&sd_free[1], 128);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 256);
    mbar_init(&ds_free[0], 1);
    mbar_init(&ds_free[1], 1);
    mbar_init(const_ready, 256);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool timed_out = false;
  static_assert(C::EW_REGS * 256 + C::CONTROL_REGS * 128 <= 168 * 384, "register split exceeds the launch");

  const bool tmem_bad = tmem_alloc_bad(tmem);  // debug builds only
  if (tmem_bad) {
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && NT > 0) {
        if (C::FUSED_DQ) tma_prefetch_desc(&tmdQacc);
        mbar_arrive_expect_tx(fix_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          tma_load_3d(sFix + cb * C::BLOCK_BYTES, &tmK, fix_full, cb * 64, j0, bh);
          tma_load_3d(sFix + C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmV, fix_full, cb * 64, j0, bh);
        }
        int issued = 0;
        for (int t = 0; t < NT; ++t) {
          const int st = t % C::NSTAGE;
          if (!mbar_wait_bounded(&empty[st], ((uint32_t)(t / C::NSTAGE) & 1u) ^ 1u, abort_flag, &timed_out)) break;
          uint8_t* dst = sSt + st * C::STAGE_BYTES;
          const int q0 = (t_first + t) * 128;
          mbar_arrive_expect_tx(&full[st], 2 * C::TILE_BYTES + (aug ? 4096 : 1024));
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_3d(dst + cb * C::BLOCK_BYTES, &tmQ, &full[st], cb * 64, q0, bh);
            tma_load_3d(dst + C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmdO, &full[st], cb * 64, q0, bh);
          }
          if (aug) {
            bulk_load(dst + 2 * C::TILE_BYTES, p.aug + ((size_t)bh * (p.n_q_pad / 128) + (t_first + t)) * 4096, 4096,
                      &full[st]);
          } else {
            const size_t v0 = (size_t)bh * p.n_q_pad + q0;
            bulk_load(dst + 2 * C::TILE_BYTES, p.L2 + v0, 512, &full[st]);
            bulk_load(dst + 2 * C::TILE_BYTES + 512, p.Dvec + v0, 512, &full[st]);
          }
          issued = t + 1;
        }
        if (*abort_flag) {  // let the copies in flight land before the CTA exits
          mbar_wait_drain(fix_full, 0);
          for (int t = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); t < issued; ++t)
            mbar_wait_drain(&full[t % C::NSTAGE], (uint32_t)(t / C::NSTAGE) & 1u);
        }
      }
    } else if (warp == C::MMA_WARP || (C::TWO_ISSUERS && warp == C::MMA_WARP + 1)) {
      // ------------------------------------------------------------ MMA issuer(s)
      const int role = warp - C::MMA_WARP;  // with two issuers: 0 S / dP, 1 gradients
      if (lane == 0 && NT > 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);  // K or V (K-major) x 64 rows of Q or dO
        constexpr uint32_t idA = idesc_bf16_f32(128, D, false, true);    // P^T or dS^T (TMEM) x dO or Q (MN-major)
        const uint32_t fix = smem_u32(sFix), st0 = smem_u32(sSt);
        const uint64_t dK = smem_desc_sw128(fix, 16, 1024);
        const uint64_t dV = smem_desc_sw128(fix + C::TILE_BYTES, 16, 1024);
        auto wait_bar = [&](uint64_t* bar, int phase) {
          const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
          if (r) tc_fence_after_sync();  // the elementwise warps' TMEM stores precede the products
          return r;
        };
        // Query tile t is taken in two halves of 64 rows; half h's S^T and dP^T go to columns
        // [64 h, 64 h + 64) of their regions, where warpgroup h reads them.
        auto issue_sdp = [&](int t, int h) {  // S^T_h = K Q_h^T, dP^T_h = V dO_h^T
          const uint32_t sq = st0 + (t % C::NSTAGE) * C::STAGE_BYTES + h * 8192;  // 64 rows in
          const uint64_t dQk = smem_desc_sw128(sq, 16, 1024), dOk = smem_desc_sw128(sq + C::TILE_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = (uint64_t)((((kk >> 2) * C::BLOCK_BYTES) + (kk & 3) * 32) >> 4);
            if (C::FIX_IN_TMEM) {  // K, V from TMEM: 16 keys' columns are 8 TMEM columns of bf16 pairs
              mma_ts(tmem + C::COL_S + 64 * h, tmem + C::COL_FIX + kk * 8, dQk + o, idS, kk > 0 ? 1u : 0u);
              mma_ts(tmem + C::COL_DP + 64 * h, tmem + C::COL_FIX + 32 + kk * 8, dOk + o, idS, kk > 0 ? 1u : 0u);
            } else {
              mma_ss(tmem + C::COL_S + 64 * h, dK + o, dQk + o, idS, kk > 0 ? 1u : 0u);
              mma_ss(tmem + C::COL_DP + 64 * h, dV + o, dOk + o, idS, kk > 0 ? 1u : 0u);
            }
          }
          if (aug) {  // + ones x the half's term images (S: images 0, 1; dP: images 2, 3), MN-major
            const uint32_t img = st0 + (t % C::NSTAGE) * C::STAGE_BYTES + 2 * C::TILE_BYTES + h * 1024;
            const uint32_t ones = smem_u32(smem + C::ONES_OFF), zero = smem_u32(smem + C::ZERO_OFF);
            const uint64_t dOnes = smem_desc_sw128(ones, 1024, zero - ones);
            constexpr uint32_t idAug = idesc_bf16_f32(128, 64, true, true);
            mma_ss(tmem + C::COL_S + 64 * h, dOnes, smem_desc_sw128(img, 1024, zero - img), idAug, 1u);
            mma_ss(tmem + C::COL_DP + 64 * h, dOnes, smem_desc_sw128(img + 2048, 1024, zero - img - 2048), idAug, 1u);
          }
          tc_commit(&s_full[h]);
        };
        auto issue_grad = [&](int t, int h) {  // dV += P^T_h dO_h, dK += dS^T_h Q_h (64 query rows)
          const uint32_t sq = st0 + (t % C::NSTAGE) * C::STAGE_BYTES;
          const uint64_t dOm = smem_desc_sw128(sq + C::TILE_BYTES, C::BLOCK_BYTES, 1024);  // MN-major views
          const uint64_t dQm = smem_desc_sw128(sq, C::BLOCK_BYTES, 1024);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * h + k4;
            const uint32_t acc = (t > 0 || kk > 0) ? 1u : 0u;
            const uint64_t ob = (uint64_t)((kk * 2048) >> 4);
            mma_ts(tmem + C::COL_A, tmem + C::COL_S + bwd_pair_col(kk), dOm + ob, idA, acc);
            mma_ts(tmem + C::COL_B, tmem + C::COL_DP + bwd_pair_col(kk), dQm + ob, idA, acc);
          }
        };
        // fused dQ: dQ_t = dS_t K, this key tile's share of query tile t's dQ, fresh in TMEM.  A is
        // dS (M = 128 queries, K = 128 keys) read MN-major from the buffer of dS^T rows (two
        // 64-query blocks 16 KB apart); B is K (N = d, K = keys), MN-major like V in the forward.
        constexpr uint32_t idQ = idesc_bf16_f32(128, D, true, true);
        const uint64_t dKm = smem_desc_sw128(fix, C::BLOCK_BYTES, 1024);
        auto issue_dq = [&](int t) {
          const uint64_t dDSm = smem_desc_sw128(smem_u32(sDS + (t & 1) * C::DS_BYTES), C::BLOCK_BYTES, 1024);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint64_t o = (uint64_t)((kk * 2048) >> 4);
            mma_ss(tmem + C::COL_DQ, dDSm + o, dKm + o, idQ, kk > 0 ? 1u : 0u);
          }
        };
        // Half h of tile t + 1 starts as soon as warpgroup h has finished half h of tile t, so one
        // warpgroup's elementwise pass overlaps the other's and the tensor core's products.
        bool ok = true;
        if (!C::TWO_ISSUERS) {
          ok = wait_bar(fix_full, 0) && wait_bar(&full[0], 0) && (!C::FIX_IN_TMEM || wait_bar(fix_tmem, 0)) &&
               (!aug || wait_bar(const_ready, 0));
          if (ok) {
            issue_sdp(0, 0);
            issue_sdp(0, 1);
          }
          for (int t = 0; ok && t < NT; ++t) {
            for (int h = 0; ok && h < 2; ++h) {
              if (!(ok = wait_bar(&p_full[h], t))) break;
              issue_grad(t, h);
              if (h == 1) tc_commit(&empty[t % C::NSTAGE]);
              if (t + 1 < NT) {
                if (h == 0 && !(ok = wait_bar(&full[(t + 1) % C::NSTAGE], (t + 1) / C::NSTAGE))) break;
                issue_sdp(t + 1, h);
              }
            }
            if (C::FUSED_DQ && ok) {  // both halves' dS_t are in the buffer; dQ_(t-1) has been read out
              if (t > 0 && !(ok = wait_bar(dq_free, t - 1))) break;
              issue_dq(t);
              tc_commit(dq_full);
              tc_commit(&ds_free[t & 1]);
            }
          }
          if (ok) tc_commit(o_full);
        } else if (role == 0) {  // S / dP: half h of tile t once the gradient products of half h of t - 1 are done
          ok = wait_bar(fix_full, 0) && (!C::FIX_IN_TMEM || wait_bar(fix_tmem, 0)) && (!aug || wait_bar(const_ready, 0));
          for (int t = 0; ok && t < NT; ++t)
            for (int h = 0; ok && h < 2; ++h) {
              if (h == 0 && !(ok = wait_bar(&full[t % C::NSTAGE], t / C::NSTAGE))) break;
              if (t > 0 && !(ok = wait_bar(&grad_done[h], t - 1))) break;
              issue_sdp(t, h);
            }
        } else {  // gradients: half h of tile t once its elementwise pass is done
          for (int t = 0; ok && t < NT; ++t)
            for (int h = 0; ok && h < 2; ++h) {
              if (!(ok = wait_bar(&p_full[h], t))) break;
              issue_grad(t, h);
              tc_commit(&grad_done[h]);
              if (h == 1) tc_commit(&empty[t % C::NSTAGE]);
            }
          if (ok) tc_commit(o_full);
        }
        tc_commit(&drain[role]);
        mbar_wait_drain(&drain[role], 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::EW_REGS));
    // ------------------------------------------------------- elementwise + epilogue
    const int w = warp >> 2;           // column half of the tile
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = key within the tile
    const int key = j0 + row;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale_log2;
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, int phase) {
      const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      return __all_sync(0xffffffffu, r);
    };
    if (C::FIX_IN_TMEM && NT > 0 && (ok = wait_warp(fix_full, 0))) {
      // row `row` of fixed tile w into this warp's TMEM lanes, 32 columns of bf16 pairs: the
      // 128-byte rows sit in 1 KB atoms of eight, their 16-byte chunks permuted by the
      // 128-byte swizzle (chunk c of row r at position c ^ (r % 8))
      const uint8_t* rp = sFix + w * C::TILE_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 q4 = *reinterpret_cast<const uint4*>(rp + ((c ^ (row & 7)) << 4));
        v[4 * c] = q4.x, v[4 * c + 1] = q4.y, v[4 * c + 2] = q4.z, v[4 * c + 3] = q4.w;
      }
      tmem_st_32x32b_x32(tmem + C::COL_FIX + 32u * (uint32_t)w + lane_base, v);
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(fix_tmem);
    }
    if (aug) {  // the ones block (rows 0-2 of both 64-key images) and the zeros, 16 bytes per thread
      const int i = threadIdx.x;  // 0 .. 255
      const uint32_t one2 = 0x3F803F80u;  // two bf16 ones
      const bool ones_row = i < 128 && ((i & 63) >> 3) < 3;  // byte (i & 63) * 16 of image i >> 6: row (i & 63) / 8
      *reinterpret_cast<uint4*>(smem + C::ONES_OFF + i * 16) =
          ones_row ? make_uint4(one2, one2, one2, one2) : make_uint4(0u, 0u, 0u, 0u);
      if (i >= 128) *reinterpret_cast<uint4*>(smem + C::ZERO_OFF + (i - 128) * 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      mbar_arrive(const_ready);
    }
    // Fused dQ: query tile tt's dQ_tt leaves TMEM through this warpgroup's staging buffer (its 32 of
    // the D columns, rows = queries, 128-byte swizzle) and one TMA reduce-add into the fp32
    // accumulator, issued by the warpgroup's first thread.  The warpgroup's four warps agree on
    // every drain with a barrier vote, so a failed wait in any of them makes all of them skip it
    // (and the later ones): each warp takes part in exactly NT votes, its share of every drain,
    // whatever fails, and none is left waiting at a named barrier.
    const int wg_bar = 1 + w;  // named barrier of this warpgroup (128 threads)
    const bool wg_leader = (threadIdx.x & 127) == 0;
    int n_votes = 0;
    auto drain_dq = [&](int tt, bool can) -> bool {
      const bool r = can && mbar_wait_bounded(dq_full, (uint32_t)tt & 1u, abort_flag, &timed_out);
      if (wg_leader) bulk_wait_group_read_all();  // the previous reduce has read the staging buffer
      ++n_votes;
      if (named_bar_any(wg_bar, 128, !r)) return false;
      tc_fence_after_sync();
      uint32_t v[32];
      tmem_ld_32x32b_x32(tmem + C::COL_DQ + 32u * (uint32_t)w + lane_base, v);
      tmem_wait_ld();
      reg_fence(v);
      tc_fence_before_sync();
      mbar_arrive(dq_free);
      uint8_t* rp = sStg[w] + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(rp + ((c ^ (row & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      fence_proxy_async_smem();
      named_bar_sync(wg_bar, 128);
      if (wg_leader) {
        tma_reduce_add_3d(&tmdQacc, sStg[w], 32 * w, (t_first + tt) * 128, bh);
        bulk_commit_group();
      }
      return true;
    };
    for (int t = 0; ok && t < NT; ++t) {
      const int st = t % C::NSTAGE;
      const float* vL2 = reinterpret_cast<const float*>(sSt + st * C::STAGE_BYTES + 2 * C::TILE_BYTES);
      const float* vD = vL2 + 128;
      // the stage's vectors come from the bulk copy: wait for it here too, not only through the MMAs
      // (with the term images in the products nothing of the stage is read here)
      if (!(ok = (aug || wait_warp(&full[st], t / C::NSTAGE)) && wait_warp(&s_full[w], t))) break;
      // fused dQ: the dQ product of tile t - 2 has read dS buffer t % 2 (its (t / 2 - 1)-th use)
      if (C::FUSED_DQ && t > 1 && !(ok = wait_warp(&ds_free[t & 1], t / 2 - 1))) break;
      tc_fence_after_sync();
      const int q0 = (t_first + t) * 128 + 64 * w;  // first query of this warpgroup's columns
      const bool masked = CAUSAL && (q0 + off < j0 + 127);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cbase = 64 * w + 32 * h;  // tile column of this chunk
        uint32_t s[32], dp[32];
        tmem_ld_32x32b_x32(tmem + C::COL_S + (uint32_t)cbase + lane_base, s);
        tmem_ld_32x32b_x32(tmem + C::COL_DP + (uint32_t)cbase + lane_base, dp);
        tmem_wait_ld();
        reg_fence(s);
        reg_fence(dp);
        uint32_t pp[16], ps[16];
        const int qc = q0 + 32 * h;
        if (C::AUG && aug) {  // the per-query terms are already in s and dp
          const auto zero = [](int) { return 0.f; };
          if (masked)
            bwd_elementwise(s, dp, c2, zero, zero, [&](int c) { return key <= qc + c + off; }, pp, ps);
          else
            bwd_elementwise(s, dp, c2, zero, zero, [&](int) { return true; }, pp, ps);
        } else {
          // this chunk's 32 query vectors, four per 16-byte load (every lane reads the same words)
          float l2v[32], ddv[32];
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 a = *reinterpret_cast<const float4*>(vL2 + cbase + c);
            const float4 b = *reinterpret_cast<const float4*>(vD + cbase + c);
            l2v[c] = a.x, l2v[c + 1] = a.y, l2v[c + 2] = a.z, l2v[c + 3] = a.w;
            ddv[c] = b.x, ddv[c + 1] = b.y, ddv[c + 2] = b.z, ddv[c + 3] = b.w;
          }
          if (masked)
            bwd_elementwise(s, dp, c2, [&](int c) { return l2v[c]; }, [&](int c) { return ddv[c]; },
                            [&](int c) { return key <= qc + c + off; }, pp, ps);
          else
            bwd_elementwise(s, dp, c2, [&](int c) { return l2v[c]; }, [&](int c) { return ddv[c]; },
                            [&](int) { return true; }, pp, ps);
        }
        tmem_st_32x32b_x16(tmem + C::COL_S + (uint32_t)(64 * w + 16 * h) + lane_base, pp);
        tmem_st_32x32b_x16(tmem + C::COL_DP + (uint32_t)(64 * w + 16 * h) + lane_base, ps);
        if (C::FUSED_DQ) {  // and into the dS buffer: key `row`, this chunk's 32 queries (16-byte chunks 4h ..)
          uint8_t* rp = sDS + (t & 1) * C::DS_BYTES + w * C::BLOCK_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            *reinterpret_cast<uint4*>(rp + (((4 * h + i) ^ (row & 7)) << 4)) =
                make_uint4(ps[4 * i], ps[4 * i + 1], ps[4 * i + 2], ps[4 * i + 3]);
        }
      }
      tmem_wait_st();
      tc_fence_before_sync();
      if (C::FUSED_DQ) fence_proxy_async_smem();  // the dS rows are read by the tensor core
      mbar_arrive(&p_full[w]);
      if (C::FUSED_DQ && t > 0 && !(ok = drain_dq(t - 1, true))) break;
    }
    if (C::FUSED_DQ && NT > 0) {
      // the last tile's dQ, then the votes a failure left out; all reduces complete before exit
      if (n_votes < NT) ok = drain_dq(NT - 1, ok) && ok;
      while (n_votes < NT) drain_dq(n_votes, false);
      if (wg_leader) bulk_wait_group_all();
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && NT > 0) ok = wait_warp(o_full, 0);
    if (ok) {
      tc_fence_after_sync();
      // warpgroup 0 writes dV, warpgroup 1 writes dK (times scale); zeros if no query sees the tile
      const uint32_t col = w ? C::COL_B : C::COL_A;
      const float mul = w ? p.scale : 1.f;
      const bool store = key < p.n_kv;
      __nv_bfloat16* dst = (w ? p.dK : p.dV) + ((size_t)bh * p.n_kv + (store ? key : 0)) * D;
#pragma unroll 1
      for (int cb = 0; cb < D; cb += 32) {
        uint32_t o[32];
        if (NT > 0) {
          tmem_ld_32x32b_x32(tmem + col + (uint32_t)cb + lane_base, o);
          tmem_wait_ld();
          reg_fence(o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cb);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    }
  }

  if (timed_out) record_error(6 /* SDPA_ERR_DEVICE_TIMEOUT */);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------ dQ
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(384, 1)
    sdpa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                       const BwdParams p) {
  using C = BwdCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sFix = smem + C::FIX_OFF;  // Q, dO
  uint8_t* sSt = smem + C::ST_OFF;    // per stage: K, V
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* fix_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + C::NSTAGE;
  uint64_t* s_full = empty + C::NSTAGE;  // [half]
  uint64_t* p_full = s_full + 2;         // [half] = [warpgroup]
  uint64_t* grad_done = p_full + 2;      // [half]: the gradient products reading half h completed
  uint64_t* o_full = grad_done + 2;
  uint64_t* drain = o_full + 1;          // [issuer]
  uint64_t* fix_tmem = drain + 2;        // d = 64: the fixed pair has been copied into TMEM
  uint64_t* sd_free = fix_tmem + 1;      // [half] (dq): S and dP of half h are in registers
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x % p.bh_count;
  const int n_qt = (p.n_q + 127) / 128;
  const int q0 = (n_qt - 1 - (int)(blockIdx.x / p.bh_count)) * 128;  // causal: the last rows see the most keys
  const int off = p.n_kv - p.n_q;
  int T = (p.n_kv + 127) / 128;  // key tiles this query tile visits
  if (CAUSAL) {
    const int last_row = (q0 + 127 < p.n_q - 1) ? q0 + 127 : p.n_q - 1;
    const long long max_key = (long long)last_row + off;
    T = max_key < 0 ? 0 : (int)(max_key / 128) + 1 < T ? (int)(max_key / 128) + 1 : T;
  }

  if (threadIdx.x == 0) {
    mbar_init(fix_full, 1);
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(&grad_done[0], 1);
    mbar_init(&grad_done[1], 1);
    mbar_init(o_full, 1);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(fix_tmem, 256);
    mbar_init(&sd_free[0], 128);
    mbar_init(&sd_free[1], 128);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool timed_out = false;
  static_assert(C::EW_REGS * 256 + C::CONTROL_REGS * 128 <= 168 * 384, "register split exceeds the launch");

  const bool tmem_bad = tmem_alloc_bad(tmem);  // debug builds only
  if (tmem_bad) {
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && T > 0) {
        mbar_arrive_expect_tx(fix_full, 2 * C::TILE_BYTES);
#pragma unroll
        for (int cb = 0; cb < D / 64; ++cb) {
          tma_load_3d(sFix + cb * C::BLOCK_BYTES, &tmQ, fix_full, cb * 64, q0, bh);
          tma_load_3d(sFix + C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmdO, fix_full, cb * 64, q0, bh);
        }
        int issued = 0;
        for (int j = 0; j < T; ++j) {
          const int st = j % C::NSTAGE;
          if (!mbar_wait_bounded(&empty[st], ((uint32_t)(j / C::NSTAGE) & 1u) ^ 1u, abort_flag, &timed_out)) break;
          uint8_t* dst = sSt + st * C::STAGE_BYTES;
          mbar_arrive_expect_tx(&full[st], 2 * C::TILE_BYTES);
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb) {
            tma_load_3d(dst + cb * C::BLOCK_BYTES, &tmK, &full[st], cb * 64, j * 128, bh);
            tma_load_3d(dst + C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmV, &full[st], cb * 64, j * 128, bh);
          }
          issued = j + 1;
        }
        if (*abort_flag) {
          mbar_wait_drain(fix_full, 0);
          for (int j = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); j < issued; ++j)
            mbar_wait_drain(&full[j % C::NSTAGE], (uint32_t)(j / C::NSTAGE) & 1u);
        }
      }
    } else if (warp == C::MMA_WARP || (C::TWO_ISSUERS && warp == C::MMA_WARP + 1)) {
      // ------------------------------------------------------------ MMA issuer(s)
      const int role = warp - C::MMA_WARP;  // with two issuers: 0 S / dP, 1 gradients
      if (lane == 0 && T > 0) {
        constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false);  // Q or dO (K-major) x 64 rows of K or V
        constexpr uint32_t idA = idesc_bf16_f32(128, D, false, true);    // dS (TMEM) x K (MN-major)
        const uint32_t fix = smem_u32(sFix), st0 = smem_u32(sSt);
        const uint64_t dQk = smem_desc_sw128(fix, 16, 1024);
        const uint64_t dOk = smem_desc_sw128(fix + C::TILE_BYTES, 16, 1024);
        auto wait_bar = [&](uint64_t* bar, int phase) {
          const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
          if (r) tc_fence_after_sync();  // the elementwise warps' TMEM stores precede the products
          return r;
        };
        auto issue_sdp = [&](int j, int h) {  // S_h = Q K_h^T, dP_h = dO V_h^T (64 keys)
          const uint32_t sk = st0 + (j % C::NSTAGE) * C::STAGE_BYTES + h * 8192;
          const uint64_t dKk = smem_desc_sw128(sk, 16, 1024), dVk = smem_desc_sw128(sk + C::TILE_BYTES, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t o = (uint64_t)((((kk >> 2) * C::BLOCK_BYTES) + (kk & 3) * 32) >> 4);
            if (C::FIX_IN_TMEM) {  // Q, dO from TMEM
              mma_ts(tmem + C::COL_S + 64 * h, tmem + C::COL_FIX + kk * 8, dKk + o, idS, kk > 0 ? 1u : 0u);
              mma_ts(tmem + C::COL_DP + 64 * h, tmem + C::COL_FIX + 32 + kk * 8, dVk + o, idS, kk > 0 ? 1u : 0u);
            } else {
              mma_ss(tmem + C::COL_S + 64 * h, dQk + o, dKk + o, idS, kk > 0 ? 1u : 0u);
              mma_ss(tmem + C::COL_DP + 64 * h, dOk + o, dVk + o, idS, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(&s_full[h]);
        };
        auto issue_grad = [&](int j, int h) {  // dQ += dS_h K_h
          const uint64_t dKm = smem_desc_sw128(st0 + (j % C::NSTAGE) * C::STAGE_BYTES, C::BLOCK_BYTES, 1024);
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int kk = 4 * h + k4;
            // dS pairs: in their own columns (32 per warpgroup) or over dP (bwd_pair_col)
            const uint32_t a_col = C::DS_SEPARATE ? C::COL_DS + (uint32_t)((kk >> 2) * 32 + (kk & 3) * 8)
                                                  : C::COL_DP + bwd_pair_col(kk);
            mma_ts(tmem + C::COL_A, tmem + a_col, dKm + (uint64_t)((kk * 2048) >> 4), idA, (j > 0 || kk > 0) ? 1u : 0u);
          }
        };
        bool ok = true;
        if (!C::TWO_ISSUERS) {
          ok = wait_bar(fix_full, 0) && wait_bar(&full[0], 0) && (!C::FIX_IN_TMEM || wait_bar(fix_tmem, 0));
          if (ok) {
            issue_sdp(0, 0);
            issue_sdp(0, 1);
          }
          for (int j = 0; ok && j < T; ++j) {
            for (int h = 0; ok && h < 2; ++h) {
              if (C::DS_SEPARATE && j + 1 < T) {  // next S / dP of half h once S, dP of half h are read
                if (h == 0 && !(ok = wait_bar(&full[(j + 1) % C::NSTAGE], (j + 1) / C::NSTAGE))) break;
                if (!(ok = wait_bar(&sd_free[h], j))) break;
                issue_sdp(j + 1, h);
              }
              if (!(ok = wait_bar(&p_full[h], j))) break;
              issue_grad(j, h);
              if (C::DS_SEPARATE) tc_commit(&grad_done[h]);
              if (h == 1) tc_commit(&empty[j % C::NSTAGE]);
              if (!C::DS_SEPARATE && j + 1 < T) {
                if (h == 0 && !(ok = wait_bar(&full[(j + 1) % C::NSTAGE], (j + 1) / C::NSTAGE))) break;
                issue_sdp(j + 1, h);
              }
            }
          }
          if (ok) tc_commit(o_full);
        } else if (role == 0) {
          ok = wait_bar(fix_full, 0) && (!C::FIX_IN_TMEM || wait_bar(fix_tmem, 0));
          for (int j = 0; ok && j < T; ++j)
            for (int h = 0; ok && h < 2; ++h) {
              if (h == 0 && !(ok = wait_bar(&full[j % C::NSTAGE], j / C::NSTAGE))) break;
              if (j > 0 && !(ok = wait_bar(C::DS_SEPARATE ? &sd_free[h] : &grad_done[h], j - 1))) break;
              issue_sdp(j, h);
            }
        } else {
          for (int j = 0; ok && j < T; ++j)
            for (int h = 0; ok && h < 2; ++h) {
              if (!(ok = wait_bar(&p_full[h], j))) break;
              issue_grad(j, h);
              tc_commit(&grad_done[h]);
              if (h == 1) tc_commit(&empty[j % C::NSTAGE]);
            }
          if (ok) tc_commit(o_full);
        }
        tc_commit(&drain[role]);
        mbar_wait_drain(&drain[role], 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::EW_REGS));
    // ------------------------------------------------------- elementwise + epilogue
    const int w = warp >> 2;                 // column half: keys [64 w, 64 w + 64) of each tile
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = query row within the tile
    const int q = q0 + row;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale_log2;
    const size_t vi = (size_t)bh * p.n_q_pad + q;  // inside the padded vectors for every lane
    // written by the pre kernel: read through L2 (this grid may start before dkdv has finished)
    const float l2 = __ldcg(p.L2 + vi);
    const float dd = __ldcg(p.Dvec + vi);
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, int phase) {
      const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      return __all_sync(0xffffffffu, r);
    };
    if (C::FIX_IN_TMEM && T > 0 && (ok = wait_warp(fix_full, 0))) {
      // row `row` of fixed tile w (Q or dO) into this warp's TMEM lanes, as in the dK/dV kernel
      const uint8_t* rp = sFix + w * C::TILE_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
      uint32_t v[32];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 q4 = *reinterpret_cast<const uint4*>(rp + ((c ^ (row & 7)) << 4));
        v[4 * c] = q4.x, v[4 * c + 1] = q4.y, v[4 * c + 2] = q4.z, v[4 * c + 3] = q4.w;
      }
      tmem_st_32x32b_x32(tmem + C::COL_FIX + 32u * (uint32_t)w + lane_base, v);
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(fix_tmem);
    }
    for (int j = 0; ok && j < T; ++j) {
      if (!(ok = wait_warp(&s_full[w], j))) break;
      tc_fence_after_sync();
      const int k0 = j * 128 + 64 * w;  // first key of this warpgroup's columns
      const bool masked = (k0 + 63 >= p.n_kv) || (CAUSAL && k0 + 63 > q0 + off);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int cbase = 64 * w + 32 * h;
        uint32_t s[32], dp[32];
        tmem_ld_32x32b_x32(tmem + C::COL_S + (uint32_t)cbase + lane_base, s);
        tmem_ld_32x32b_x32(tmem + C::COL_DP + (uint32_t)cbase + lane_base, dp);
        tmem_wait_ld();
        reg_fence(s);
        reg_fence(dp);
        if (C::DS_SEPARATE && h == 0) {
          // the last dQ product reading this warpgroup's dS columns has completed
          if (j > 0 && !(ok = wait_warp(&grad_done[w], j - 1))) break;
          tc_fence_after_sync();
        }
        if (C::DS_SEPARATE && h == 1) {
          // this warpgroup's S and dP columns are all in registers: with dS in columns of its own
          // the tensor core may overwrite them with the next key tile's S and dP
          tc_fence_before_sync();
          mbar_arrive(&sd_free[w]);
        }
        uint32_t pp[16], ps[16];
        const int kc = k0 + 32 * h;
        if (masked)
          bwd_elementwise(s, dp, c2, [&](int) { return l2; }, [&](int) { return dd; },
                          [&](int c) { return kc + c < p.n_kv && (!CAUSAL || kc + c <= q + off); }, pp, ps);
        else
          bwd_elementwise(s, dp, c2, [&](int) { return l2; }, [&](int) { return dd; }, [&](int) { return true; }, pp,
                          ps);
        const uint32_t col =
            C::DS_SEPARATE ? C::COL_DS + (uint32_t)(32 * w + 16 * h) : C::COL_DP + (uint32_t)(64 * w + 16 * h);
        tmem_st_32x32b_x16(tmem + col + lane_base, ps);
      }
      if (!ok) break;
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&p_full[w]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && T > 0) ok = wait_warp(o_full, 0);
    if (ok) {
      tc_fence_after_sync();
      // warpgroup w writes columns [w D/2, w D/2 + D/2) of this row's dQ (times scale)
      const bool store = q < p.n_q;
      __nv_bfloat16* dst = p.dQ + ((size_t)bh * p.n_q + (store ? q : 0)) * D;
#pragma unroll 1
      for (int cb = w * (D / 2); cb < (w + 1) * (D / 2); cb += 32) {
        uint32_t o[32];
        if (T > 0) {
          tmem_ld_32x32b_x32(tmem + C::COL_A + (uint32_t)cb + lane_base, o);
          tmem_wait_ld();
          reg_fence(o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint32_t v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          v[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * p.scale, __uint_as_float(o[2 * i + 1]) * p.scale);
        if (store) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cb);
#pragma unroll
          for (int i = 0; i < 4; ++i) d4[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
    }
  }

  // dkdv, before this kernel on the stream, may still be finishing (it let this one start early):
  // the stream must see both done when this grid completes.
  if (threadIdx.x == 0) griddep_wait();
  if (timed_out) record_error(6 /* SDPA_ERR_DEVICE_TIMEOUT */);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdpa
