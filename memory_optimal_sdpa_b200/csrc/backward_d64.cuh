// backward_d64.cuh -- gradients of exact SDPA at d = 64 in one tensor-core kernel (dK, dV and dQ).
//
// The same arithmetic as backward.cuh (agents-report.net MoA article, "implementation roadmap":
// the backward pass in the memory-optimal form): per key tile j and query tile t,
//   S^T = K_j Q_t^T, dP^T = V_j dO_t^T,  P^T = 2^(S^T scale log2(e) - LSE log2(e)),
//   dS^T = P^T (dP^T - D),  dV_j += P^T dO_t,  dK_j += dS^T Q_t,  dQ_t += dS_t K_j,
// dV and dK kept in TMEM over the query tiles, dQ_t formed per tile and reduce-added in fp32 into
// a workspace by TMA (a small kernel then writes dQ = scale * that sum in bf16).
//
// What differs from the general dK/dV kernel is where the intermediates live, so that the next
// S^T / dP^T products never wait for the gradient products of the current tile:
//   TMEM  S^T [0, 128) and dP^T [128, 256) fp32 -- released as soon as the elementwise warps hold
//         them in registers; P^T (bf16 pairs) [256, 320) in columns of its own; dV [320, 384),
//         dK [384, 448), dQ_t [448, 512) fp32
//   smem  K and V of the key tile; two stages of (Q_t, dO_t, the per-query terms); dS^T of tile t
//         in buffer t % 2 (bf16, keys x queries, 128-byte swizzle), read K-major as the A operand
//         of dK and MN-major as the A operand of dQ; the fp32 staging of dQ_t for the reduce.
// The per-query terms (-LSE log2(e) / c2 for S, -D for dP) enter the S^T and dP^T products as one
// more K step (see SDPA_BWD64_AUG), so the elementwise step is P = 2^(S' c2), dS = P dP' with no
// per-column loads: those broadcast loads had cost about a fifth of the shared-memory bandwidth
// (measured 4 x 16 x 2048: 507 -> 628 TF/s).
// Warp roles (512 threads): warps 0-7 two elementwise warpgroups (warpgroup w takes query
// columns [64 w, 64 w + 64) of each tile: its "half"; thread = TMEM lane = key of the tile),
// warp 8 the TMA producer, warp 9 the issuer of S^T, dP^T and dQ and TMEM owner, warp 10 the
// issuer of the dV and dK products, warp 11 idle, warps 12-15 the dQ drain (TMEM -> staging ->
// TMA reduce-add).  Measured on 4 x 16 x 2048 (TF/s, non-causal / causal): dQ drained by the
// elementwise warps with a two-stage ring 628 / 452; drain warpgroup and three stages 663-679 /
// 474-489; dQ moved to the S issuer with N = 128 S^T, dP^T products 675 / 480.
#pragma once

#include "backward.cuh"

#ifndef SDPA_BWD64_SDP_N128
#define SDPA_BWD64_SDP_N128 1  // S^T and dP^T of both halves in N = 128 products (half the instructions)
#endif
// The per-query terms enter the S^T and dP^T products as one more K = 16 step: A is a block of
// ones (rows 0-2), B holds -LSE log2(e) / c2 and -D as three bf16 terms each (rows 0-2), so the
// accumulators come out as S^T - LSE log2(e) / c2 and dP^T - D and the elementwise step reads no
// per-column vectors from shared memory (needs scale != 0; the host takes the general kernels
// otherwise).
#ifndef SDPA_BWD64_AUG
#define SDPA_BWD64_AUG 1
#endif
// dQ_t leaves TMEM through a warpgroup of its own (warps 12-15, 512 threads) rather than through
// the elementwise warps between two tiles.
#ifndef SDPA_BWD64_DRAIN_WG
#define SDPA_BWD64_DRAIN_WG 1
#endif
// The dQ products are issued by the S^T / dP^T issuer (after the next tile's S^T, dP^T) rather
// than by the gradient issuer, which balances the two instruction streams (18 and 16 products).
#ifndef SDPA_BWD64_DQ_ON_A
#define SDPA_BWD64_DQ_ON_A 1
#endif

namespace sdpa {

struct BwdD64Cfg {
  static constexpr int D = 64;
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128 x 64 bf16 tile = one 128-byte-swizzle block
  static constexpr bool DRAIN_WG = SDPA_BWD64_DRAIN_WG;
  // Q_t, dO_t ring: three stages when the drain warpgroup stages dQ through one 16 KB image
  static constexpr int NSTAGE = DRAIN_WG ? 3 : 2;
  static constexpr int NSTG = DRAIN_WG ? 1 : 2;  // dQ staging images
  static constexpr bool AUG = SDPA_BWD64_AUG;
  static constexpr bool SDP_N128 = SDPA_BWD64_SDP_N128;
  static constexpr bool DQ_ON_A = SDPA_BWD64_DQ_ON_A;
  // per query tile after Q and dO: with AUG the four 1 KB images of the -LSE log2(e) / c2 and -D
  // terms ([S, dP] x [half]); else the vectors LSE log2(e) [128] and D [128]
  static constexpr int VEC_BYTES = AUG ? 4096 : 1024;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + VEC_BYTES;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int STG_BYTES = 128 * 32 * 4;
  static constexpr int FIX_OFF = 0;  // K, V
  static constexpr int ST_OFF = 2 * TILE_BYTES;
  static constexpr int DS_OFF = ST_OFF + NSTAGE * STAGE_BYTES;
  static constexpr int STG_OFF = DS_OFF + 2 * DS_BYTES;
  // AUG: the ones block (two 64-key images, rows 0-2 = 1) and 2 KB of zeros (rows 8-15 of every
  // augmented operand)
  static constexpr int ONES_OFF = STG_OFF + NSTG * STG_BYTES;
  static constexpr int ZERO_OFF = ONES_OFF + (AUG ? 2048 : 0);
  static constexpr int BAR_OFF = ZERO_OFF + (AUG ? 2048 : 0);
  // fix_full, full[NSTAGE], empty[NSTAGE], s_full[2], sd_free[2], p_full[2], grad_done[2], o_full,
  // drain[2], dq_full, dq_free, ds_free[2], const_ready
  static constexpr int NBAR = 1 + 2 * NSTAGE + 8 + 1 + 2 + 4 + 1;
  static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 16 + 1024;
  static constexpr int THREADS = DRAIN_WG ? 512 : 384;
  static constexpr int LAUNCH_REGS = DRAIN_WG ? 128 : 168;  // registers per thread the launch provides
  // 192 x 256 + 64 x 128 + 64 x 128 = 128 x 512 (without the drain warpgroup: 192 x 256 + 120 x 128 = 168 x 384)
  static constexpr int EW_REGS = 192;
  static constexpr int CONTROL_REGS = DRAIN_WG ? 64 : 120;
  static constexpr int DRAIN_REGS = 64;
  static constexpr int DRAIN_WARP0 = 12;
  static constexpr int LOAD_WARP = 8;
  static constexpr int SDP_WARP = 9;
  static constexpr int GRAD_WARP = 10;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_P = 256, COL_DV = 320, COL_DK = 384, COL_DQ = 448;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(DS_OFF % 1024 == 0 && STG_OFF % 1024 == 0 && ONES_OFF % 1024 == 0 && ZERO_OFF % 1024 == 0 &&
                    STAGE_BYTES % 1024 == 0,
                "swizzled buffers need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Elementwise step of 32 query columns (the tile's columns c0 .. c0 + 31 of this thread's key
// row): P = 2^(S c2 - l2), dS = P (dP - D), zero where `keep` is false; the row's LSE log2(e)
// and D values are read from the stage's vectors four at a time.
template <class KEEP>
__device__ __forceinline__ void bwd64_chunk(const uint32_t* s, const uint32_t* dp, float c2, const float* vL2,
                                            const float* vD, KEEP keep, uint32_t (&pp)[16], uint32_t (&ps)[16]) {
#pragma unroll
  for (int c4 = 0; c4 < 32; c4 += 4) {
    const float4 l4 = *reinterpret_cast<const float4*>(vL2 + c4);
    const float4 d4 = *reinterpret_cast<const float4*>(vD + c4);
    const float l2v[4] = {l4.x, l4.y, l4.z, l4.w}, ddv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int i = 0; i < 4; i += 2) {
      float pr[2], dr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = c4 + i + h;
        float e = sm100::ex2_approx(__uint_as_float(s[c]) * c2 - l2v[i + h]);
        if (!keep(c)) e = 0.f;
        pr[h] = e;
        dr[h] = e * (__uint_as_float(dp[c]) - ddv[i + h]);
      }
      pp[(c4 + i) >> 1] = sm100::pack_bf16x2(pr[0], pr[1]);
      ps[(c4 + i) >> 1] = sm100::pack_bf16x2(dr[0], dr[1]);
    }
  }
}

// The same with the per-column terms already inside s and dp (AUG): P = 2^(s c2), dS = P dp.
template <class KEEP>
__device__ __forceinline__ void bwd64_chunk_aug(const uint32_t* s, const uint32_t* dp, float c2, KEEP keep,
                                                uint32_t (&pp)[16], uint32_t (&ps)[16]) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float pr[2], dr[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float e = sm100::ex2_approx(__uint_as_float(s[i + h]) * c2);
      if (!keep(i + h)) e = 0.f;
      pr[h] = e;
      dr[h] = e * __uint_as_float(dp[i + h]);
    }
    pp[i >> 1] = sm100::pack_bf16x2(pr[0], pr[1]);
    ps[i >> 1] = sm100::pack_bf16x2(dr[0], dr[1]);
  }
}

template <bool CAUSAL>
__global__ void __launch_bounds__(BwdD64Cfg::THREADS, 1)
    sdpa_bwd_d64_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
                        const __grid_constant__ CUtensorMap tmdQacc, const BwdParams p) {
  using C = BwdD64Cfg;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sFix = smem + C::FIX_OFF;  // K, V
  uint8_t* sSt = smem + C::ST_OFF;    // per stage: Q, dO, LSE log2(e) [128], D [128]
  uint8_t* sDS = smem + C::DS_OFF;    // [tile % 2] dS^T
  uint8_t* sStg = smem + C::STG_OFF;  // [warpgroup] dQ staging
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* fix_full = bars;
  uint64_t* full = fix_full + 1;            // [stage]
  uint64_t* empty = full + C::NSTAGE;       // [stage]
  uint64_t* s_full = empty + C::NSTAGE;     // [half]: S^T and dP^T of the half are in TMEM
  uint64_t* sd_free = s_full + 2;           // [half]: ... and in the elementwise warps' registers
  uint64_t* p_full = sd_free + 2;           // [half]: P^T in TMEM and dS^T in shared memory
  uint64_t* grad_done = p_full + 2;         // [half]: the dV and dK products of the half completed
  uint64_t* o_full = grad_done + 2;         // dV and dK complete
  uint64_t* drain = o_full + 1;             // [issuer]
  uint64_t* dq_full = drain + 2;            // dQ_t is in TMEM
  uint64_t* dq_free = dq_full + 1;          // the elementwise warps have read dQ_t
  uint64_t* ds_free = dq_free + 1;          // [buffer]: the products reading dS^T buffer t % 2 completed
  uint64_t* const_ready = ds_free + 2;      // AUG: the ones and zero blocks are written
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  uint32_t* ds_count = tmem_slot + 2;  // DQ_ON_A: elementwise warps that have written their dS rows

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
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s_full[h], 1);
      mbar_init(&sd_free[h], 128);
      mbar_init(&p_full[h], 128);
      mbar_init(&grad_done[h], 1);
      mbar_init(&drain[h], 1);
      mbar_init(&ds_free[h], C::DQ_ON_A ? 2 : 1);  // the dK and dQ products of the buffer's tile
    }
    mbar_init(o_full, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, C::DRAIN_WG ? 128 : 256);
    mbar_init(const_ready, 256);
    *abort_flag = 0;
    *ds_count = 0;
    fence_mbar_init();
  }
  if (warp == C::SDP_WARP) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool timed_out = false;
  static_assert(C::EW_REGS * 256 + C::CONTROL_REGS * 128 + (C::DRAIN_WG ? C::DRAIN_REGS * 128 : 0) <=
                    C::LAUNCH_REGS * C::THREADS,
                "register split exceeds the launch");

  const bool tmem_bad = tmem_alloc_bad(tmem);  // debug builds only
  if (tmem_bad) {
  } else if (C::DRAIN_WG && warp >= C::DRAIN_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::DRAIN_REGS));
    // ------------------------------------------------------------ dQ drain warpgroup
    // dQ_t (TMEM lanes = the tile's queries, 64 fp32 columns), 32 columns at a time, through one
    // staging image and a TMA reduce-add into the fp32 accumulator issued by the warpgroup's first
    // thread.
    // The four warps agree on every drain with a barrier vote (named barrier 3), so a failed wait
    // in any of them makes all of them skip it and the later ones: each takes part in exactly NT
    // votes whatever fails, and none is left at a named barrier.
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const bool leader = threadIdx.x == 32 * C::DRAIN_WARP0;
    int n_votes = 0;
    auto drain = [&](int tt, bool can) -> bool {
      const bool r = can && mbar_wait_bounded(dq_full, (uint32_t)tt & 1u, abort_flag, &timed_out);
      if (leader) bulk_wait_group_read_all();  // the previous reduces have read the staging images
      ++n_votes;
      if (named_bar_any(3, 128, !r)) return false;
      tc_fence_after_sync();
      uint8_t* rp = sStg + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + C::COL_DQ + 32u * (uint32_t)c + lane_base, v);
        tmem_wait_ld();
        reg_fence(v);
        if (c == 1) {  // dQ_t has left TMEM: the next dQ product may overwrite it
          tc_fence_before_sync();
          mbar_arrive(dq_free);
          if (leader) bulk_wait_group_read_all();  // the first half's reduce has read the image
          named_bar_sync(3, 128);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(rp + ((k ^ (row & 7)) << 4)) = make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        fence_proxy_async_smem();
        named_bar_sync(3, 128);
        if (leader) {
          tma_reduce_add_3d(&tmdQacc, sStg, 32 * c, (t_first + tt) * 128, bh);
          bulk_commit_group();
        }
      }
      return true;
    };
    bool ok = true;
    for (int t = 0; ok && t < NT; ++t) ok = drain(t, true);
    while (n_votes < NT) drain(n_votes, false);
    if (leader) bulk_wait_group_all();  // every reduce has completed before the CTA exits
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && NT > 0) {
        tma_prefetch_desc(&tmdQacc);
        mbar_arrive_expect_tx(fix_full, 2 * C::TILE_BYTES);
        tma_load_3d(sFix, &tmK, fix_full, 0, j0, bh);
        tma_load_3d(sFix + C::TILE_BYTES, &tmV, fix_full, 0, j0, bh);
        int issued = 0;
        for (int t = 0; t < NT; ++t) {
          const int st = t % C::NSTAGE;
          if (!mbar_wait_bounded(&empty[st], ((uint32_t)(t / C::NSTAGE) & 1u) ^ 1u, abort_flag, &timed_out)) break;
          uint8_t* dst = sSt + st * C::STAGE_BYTES;
          const int q0 = (t_first + t) * 128;
          mbar_arrive_expect_tx(&full[st], 2 * C::TILE_BYTES + C::VEC_BYTES);
          tma_load_3d(dst, &tmQ, &full[st], 0, q0, bh);
          tma_load_3d(dst + C::TILE_BYTES, &tmdO, &full[st], 0, q0, bh);
          if (C::AUG) {
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
    } else if (warp == C::SDP_WARP || warp == C::GRAD_WARP) {
      // ------------------------------------------------------------ MMA issuers
      const int role = warp - C::SDP_WARP;  // 0: S^T and dP^T, 1: dV, dK, dQ
      if (lane == 0 && NT > 0) {
        auto wait_bar = [&](uint64_t* bar, int phase) {
          const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
          if (r) tc_fence_after_sync();  // the elementwise warps' TMEM and shared-memory writes precede the products
          return r;
        };
        const uint32_t fix = smem_u32(sFix), st0 = smem_u32(sSt), ds0 = smem_u32(sDS);
        bool ok = true;
        // dQ_t = dS_t K (M = 128 queries, N = d, K = 128 keys): dS read MN-major from dS buffer t % 2
        // (two 64-query blocks 16 KB apart), K MN-major like V in the forward.
        constexpr uint32_t idQ = idesc_bf16_f32(128, 64, true, true);
        const uint64_t dKm = smem_desc_sw128(fix, C::TILE_BYTES, 1024);
        auto issue_dq = [&](int t) {
          const uint64_t dSm = smem_desc_sw128(ds0 + (uint32_t)((t & 1) * C::DS_BYTES), C::TILE_BYTES, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t o = (uint64_t)((kk * 2048) >> 4);  // 16 keys
            mma_ss(tmem + C::COL_DQ, dSm + o, dKm + o, idQ, kk > 0 ? 1u : 0u);
          }
          tc_commit(dq_full);
          tc_commit(&ds_free[t & 1]);
        };
        if (role == 0) {
          // S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = the tile's 128 queries or the 64 of
          // half h, K = d): K, V and the stage's Q, dO rows all K-major.  With SDPA_BWD64_DQ_ON_A
          // this issuer also forms dQ_(t-1) right after S^T, dP^T of tile t.
          constexpr uint32_t idS = idesc_bf16_f32(128, 64, false, false), idS2 = idesc_bf16_f32(128, 128, false, false);
          const uint64_t dK = smem_desc_sw128(fix, 16, 1024), dV = smem_desc_sw128(fix + C::TILE_BYTES, 16, 1024);
          ok = wait_bar(fix_full, 0) && (!C::AUG || wait_bar(const_ready, 0));
          // AUG step: A = the ones block (M = 128 keys in two 64-key images 1 KB apart, MN-major),
          // B = the tile's term images (N = queries, MN-major); rows 8-15 of both read the zeros
          constexpr uint32_t idAug1 = idesc_bf16_f32(128, 64, true, true), idAug2 = idesc_bf16_f32(128, 128, true, true);
          const uint32_t ones = smem_u32(smem + C::ONES_OFF), zero = smem_u32(smem + C::ZERO_OFF);
          const uint64_t dOnes = smem_desc_sw128(ones, 1024, zero - ones);
          auto aug_desc = [&](uint32_t img) { return smem_desc_sw128(img, 1024, zero - img); };
          // dS_t of both halves in shared memory (eight elementwise warps per tile: a count, since
          // this issuer reads it up to a tile late) and dQ_(t-1) out of TMEM
          auto dq_ready = [&](int t) {
            bool r = count_wait_bounded(ds_count, 8u * (uint32_t)(t + 1), abort_flag, &timed_out);
            if (r) tc_fence_after_sync();
            if (r && t > 0) r = wait_bar(dq_free, t - 1);
            return r;
          };
          for (int t = 0; ok && t < NT; ++t) {
            const int st = t % C::NSTAGE;
            if (!(ok = wait_bar(&full[st], t / C::NSTAGE))) break;
            if (C::SDP_N128) {  // one N = 128 product per operand step, after both halves of t - 1 are read
              if (t > 0 && !(ok = wait_bar(&sd_free[0], t - 1) && wait_bar(&sd_free[1], t - 1))) break;
              const uint32_t sq = st0 + st * C::STAGE_BYTES;
              const uint64_t dQk = smem_desc_sw128(sq, 16, 1024), dOk = smem_desc_sw128(sq + C::TILE_BYTES, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t o = (uint64_t)((kk * 32) >> 4);
                mma_ss(tmem + C::COL_S, dK + o, dQk + o, idS2, kk > 0 ? 1u : 0u);
                mma_ss(tmem + C::COL_DP, dV + o, dOk + o, idS2, kk > 0 ? 1u : 0u);
              }
              if (C::AUG) {  // images [S h0, S h1, dP h0, dP h1]: one N = 128 step each
                const uint32_t img = sq + 2 * C::TILE_BYTES;
                mma_ss(tmem + C::COL_S, dOnes, aug_desc(img), idAug2, 1u);
                mma_ss(tmem + C::COL_DP, dOnes, aug_desc(img + 2048), idAug2, 1u);
              }
              tc_commit(&s_full[0]);
              tc_commit(&s_full[1]);
            } else {
              for (int h = 0; ok && h < 2; ++h) {
                if (t > 0 && !(ok = wait_bar(&sd_free[h], t - 1))) break;  // half h of tile t - 1 is in registers
                const uint32_t sq = st0 + st * C::STAGE_BYTES + h * 8192;  // query rows 64 h ..
                const uint64_t dQk = smem_desc_sw128(sq, 16, 1024), dOk = smem_desc_sw128(sq + C::TILE_BYTES, 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t o = (uint64_t)((kk * 32) >> 4);
                  mma_ss(tmem + C::COL_S + 64 * h, dK + o, dQk + o, idS, kk > 0 ? 1u : 0u);
                  mma_ss(tmem + C::COL_DP + 64 * h, dV + o, dOk + o, idS, kk > 0 ? 1u : 0u);
                }
                if (C::AUG) {
                  const uint32_t img = st0 + st * C::STAGE_BYTES + 2 * C::TILE_BYTES + h * 1024;
                  mma_ss(tmem + C::COL_S + 64 * h, dOnes, aug_desc(img), idAug1, 1u);
                  mma_ss(tmem + C::COL_DP + 64 * h, dOnes, aug_desc(img + 2048), idAug1, 1u);
                }
                tc_commit(&s_full[h]);
              }
              if (!ok) break;
            }
            if (C::DQ_ON_A && t > 0) {
              if (!(ok = dq_ready(t - 1))) break;
              issue_dq(t - 1);
            }
          }
          if (C::DQ_ON_A && ok && (ok = dq_ready(NT - 1))) issue_dq(NT - 1);
        } else {
          // dV += P^T_h dO_h (A = P^T from TMEM), dK += dS^T_h Q_h (A = dS^T K-major from shared
          // memory), M = 128 keys, N = d, K = the 64 queries of half h; dO_h, Q_h MN-major.  Then
          // (without SDPA_BWD64_DQ_ON_A) dQ_t.
          constexpr uint32_t idG = idesc_bf16_f32(128, 64, false, true);
          for (int t = 0; ok && t < NT; ++t) {
            const int st = t % C::NSTAGE;
            const uint32_t sq = st0 + st * C::STAGE_BYTES;
            const uint64_t dQm = smem_desc_sw128(sq, C::TILE_BYTES, 1024), dOm = smem_desc_sw128(sq + C::TILE_BYTES, C::TILE_BYTES, 1024);
            const uint32_t dsb = ds0 + (uint32_t)((t & 1) * C::DS_BYTES);
            for (int h = 0; ok && h < 2; ++h) {
              if (!(ok = wait_bar(&p_full[h], t))) break;
              const uint64_t dSk = smem_desc_sw128(dsb + h * C::TILE_BYTES, 16, 1024);
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4) {
                const uint32_t acc = (t > 0 || h > 0 || k4 > 0) ? 1u : 0u;
                const uint64_t ob = (uint64_t)((((4 * h + k4) * 2048)) >> 4);  // 16 query rows
                mma_ts(tmem + C::COL_DV, tmem + C::COL_P + 32 * h + 8 * k4, dOm + ob, idG, acc);
                mma_ss(tmem + C::COL_DK, dSk + (uint64_t)((k4 * 32) >> 4), dQm + ob, idG, acc);
              }
              tc_commit(&grad_done[h]);
              if (h == 1) {
                tc_commit(&empty[st]);
                if (C::DQ_ON_A) tc_commit(&ds_free[t & 1]);  // with the S issuer's commit after dQ_t
              }
            }
            if (!ok) break;
            if (!C::DQ_ON_A) {
              if (t > 0 && !(ok = wait_bar(dq_free, t - 1))) break;  // dQ_(t-1) has left TMEM
              issue_dq(t);
            }
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
    const int w = warp >> 2;                 // query half of every tile
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = key within the tile
    const int key = j0 + row;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale_log2;
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, int phase) {
      const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      return __all_sync(0xffffffffu, r);
    };
    // dQ_tt leaves TMEM through this warpgroup's staging buffer (its 32 of the 64 columns, rows =
    // queries, 128-byte swizzle) and one TMA reduce-add into the fp32 accumulator, issued by the
    // warpgroup's first thread.  The warpgroup's four warps agree on every drain with a barrier
    // vote, so a failed wait in any of them makes all of them skip it (and the later ones): each
    // warp takes part in exactly NT votes whatever fails, and none is left at a named barrier.
    const int wg_bar = 1 + w;  // named barrier of this warpgroup (128 threads)
    const bool wg_leader = (threadIdx.x & 127) == 0;
    uint8_t* stg = sStg + w * C::STG_BYTES;
    int n_votes = 0;
    if (C::AUG) {  // the ones block (rows 0-2 of both 64-key images) and the zeros, 16 bytes per thread
      const int i = threadIdx.x;  // 0 .. 255
      const uint32_t one2 = 0x3F803F80u;  // two bf16 ones
      const bool ones_row = i < 128 && ((i & 63) >> 3) < 3;  // byte (i & 63) * 16 of image i >> 6: row (i & 63) / 8
      *reinterpret_cast<uint4*>(smem + C::ONES_OFF + i * 16) =
          ones_row ? make_uint4(one2, one2, one2, one2) : make_uint4(0u, 0u, 0u, 0u);
      if (i >= 128) *reinterpret_cast<uint4*>(smem + C::ZERO_OFF + (i - 128) * 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      mbar_arrive(const_ready);
    }
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
      uint8_t* rp = stg + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(rp + ((c ^ (row & 7)) << 4)) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      fence_proxy_async_smem();
      named_bar_sync(wg_bar, 128);
      if (wg_leader) {
        tma_reduce_add_3d(&tmdQacc, stg, 32 * w, (t_first + tt) * 128, bh);
        bulk_commit_group();
      }
      return true;
    };
    for (int t = 0; ok && t < NT; ++t) {
      const int st = t % C::NSTAGE;
      const float* vL2 = reinterpret_cast<const float*>(sSt + st * C::STAGE_BYTES + 2 * C::TILE_BYTES) + 64 * w;
      const float* vD = vL2 + 128;
      // the stage's vectors (without AUG) come from the bulk copy: wait for it here too, not only
      // through the MMAs
      if (!(ok = (C::AUG || wait_warp(&full[st], t / C::NSTAGE)) && wait_warp(&s_full[w], t))) break;
      tc_fence_after_sync();
      uint32_t s[64], dp[64];
      tmem_ld_32x32b_x32(tmem + C::COL_S + 64u * (uint32_t)w + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
      tmem_ld_32x32b_x32(tmem + C::COL_S + 64u * (uint32_t)w + 32u + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
      tmem_ld_32x32b_x32(tmem + C::COL_DP + 64u * (uint32_t)w + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&dp[0]));
      tmem_ld_32x32b_x32(tmem + C::COL_DP + 64u * (uint32_t)w + 32u + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&dp[32]));
      tmem_wait_ld();
      reg_fence(s);
      reg_fence(dp);
      tc_fence_before_sync();
      mbar_arrive(&sd_free[w]);  // the next S^T, dP^T of this half may be formed
      // P^T columns: read by the dV product of tile t - 1; dS^T buffer t % 2: read by tile t - 2's
      if (t > 0 && !(ok = wait_warp(&grad_done[w], t - 1))) break;
      if (t > 1 && !(ok = wait_warp(&ds_free[t & 1], t / 2 - 1))) break;
      tc_fence_after_sync();
      const int q0 = (t_first + t) * 128 + 64 * w;  // first query of this warpgroup's columns
      const bool masked = CAUSAL && (q0 + off < j0 + 127);
      uint8_t* drow = sDS + (t & 1) * C::DS_BYTES + w * C::TILE_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pp[16], ps[16];
        const int qc = q0 + 32 * h;
        if (C::AUG) {
          if (masked)
            bwd64_chunk_aug(s + 32 * h, dp + 32 * h, c2, [&](int c) { return key <= qc + c + off; }, pp, ps);
          else
            bwd64_chunk_aug(s + 32 * h, dp + 32 * h, c2, [&](int) { return true; }, pp, ps);
        } else if (masked) {
          bwd64_chunk(s + 32 * h, dp + 32 * h, c2, vL2 + 32 * h, vD + 32 * h, [&](int c) { return key <= qc + c + off; },
                      pp, ps);
        } else {
          bwd64_chunk(s + 32 * h, dp + 32 * h, c2, vL2 + 32 * h, vD + 32 * h, [&](int) { return true; }, pp, ps);
        }
        tmem_st_32x32b_x16(tmem + C::COL_P + (uint32_t)(32 * w + 16 * h) + lane_base, pp);
        // dS^T row `row`, queries 32 h .. 32 h + 31 of the half: 16-byte chunks 4 h .. 4 h + 3
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4*>(drow + (((4 * h + i) ^ (row & 7)) << 4)) =
              make_uint4(ps[4 * i], ps[4 * i + 1], ps[4 * i + 2], ps[4 * i + 3]);
      }
      tmem_wait_st();
      tc_fence_before_sync();
      fence_proxy_async_smem();  // the dS^T rows are read by the tensor core
      mbar_arrive(&p_full[w]);
      if (C::DQ_ON_A) {
        __syncwarp();
        if (lane == 0) red_release_add(ds_count, 1u);
      }
      if (!C::DRAIN_WG && t > 0 && !(ok = drain_dq(t - 1, true))) break;
    }
    if (!C::DRAIN_WG && NT > 0) {
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
      const uint32_t col = w ? C::COL_DK : C::COL_DV;
      const float mul = w ? p.scale : 1.f;
      const bool store = key < p.n_kv;
      __nv_bfloat16* dst = (w ? p.dK : p.dV) + ((size_t)bh * p.n_kv + (store ? key : 0)) * C::D;
#pragma unroll 1
      for (int cb = 0; cb < C::D; cb += 32) {
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
  if (warp == C::SDP_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdpa
