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
//   smem  K and V of the key tile; three stages of (Q_t, dO_t, the per-query terms); dS^T of
//         tile t in buffer t % 2 (bf16, keys x queries, 128-byte swizzle), read K-major as the A
//         operand of dK and MN-major as the A operand of dQ; the fp32 staging of dQ_t for the
//         reduce; a block of ones and a block of zeros.
// The per-query terms (-LSE log2(e) / c2 for S, -D for dP, three bf16 terms each, written by the
// preprocess kernel) enter the S^T and dP^T products as one more K = 16 step against the block of
// ones, so the elementwise step is P = 2^(S' c2), dS = P dP' with no per-column loads (those
// broadcast loads had cost about a fifth of the shared-memory bandwidth).  Needs scale != 0; the
// host takes the general kernels for scale 0.
//
// Persistent: each CTA walks work units (one (batch, head) and one 128-key tile), heaviest first
// (under a causal mask the first key tiles see the most query tiles), dealt round by round in
// alternating directions.  TMEM, barriers and the constant blocks are set up once; every per-tile
// barrier phase runs on across units (a CTA-wide tile counter), the next unit's K and V are loaded
// as soon as the unit before has issued its last product reading them, and the elementwise warps
// read dV, dK of a unit out before they release the next unit's first tile.
//
// Warp roles (512 threads): warps 0-7 two elementwise warpgroups (warpgroup w takes query
// columns [64 w, 64 w + 64) of each tile: its "half"; thread = TMEM lane = key of the tile),
// warp 8 the TMA producer, warp 9 the issuer of S^T, dP^T (N = 128, both halves) and dQ and the
// TMEM owner, warp 10 the issuer of the dV and dK products, warp 11 idle, warps 12-15 the dQ
// drain (TMEM -> staging -> TMA reduce-add).
#pragma once

#include "backward.cuh"

// K, V buffers: 1 reloads them in place after the unit's last product reading them (with three
// Q/dO stages); 2 lets the next unit's K and V load during the current unit, but leaves room for
// two stages only (measured 4 x 16 x 2048: 720 -> 648 TF/s, causal 515 -> 468).
#ifndef SDPA_BWD64_KV_BUFFERS
#define SDPA_BWD64_KV_BUFFERS 1
#endif

namespace sdpa {

struct BwdD64Cfg {
  static constexpr int D = 64;
  static constexpr int TILE_BYTES = 128 * D * 2;  // one 128 x 64 bf16 tile = one 128-byte-swizzle block
  static constexpr int NFIX = SDPA_BWD64_KV_BUFFERS;  // K, V buffers
  static constexpr int NSTAGE = NFIX == 2 ? 2 : 3;     // Q_t, dO_t ring
  static constexpr int TERM_BYTES = 4096;         // the four 1 KB term images ([S, dP] x [half])
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES + TERM_BYTES;
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int STG_BYTES = 128 * 32 * 4;
  static constexpr int FIX_OFF = 0;  // [buffer] K, V
  static constexpr int ST_OFF = NFIX * 2 * TILE_BYTES;
  static constexpr int DS_OFF = ST_OFF + NSTAGE * STAGE_BYTES;
  static constexpr int STG_OFF = DS_OFF + 2 * DS_BYTES;
  // the ones block (two 64-key images, rows 0-2 = 1) and 2 KB of zeros (rows 8-15 of every
  // operand of the term step)
  static constexpr int ONES_OFF = STG_OFF + STG_BYTES;
  static constexpr int ZERO_OFF = ONES_OFF + 2048;
  static constexpr int BAR_OFF = ZERO_OFF + 2048;
  // fix_full[NFIX], fix_free[NFIX], full[NSTAGE], empty[NSTAGE], s_full[2], sd_free[2], p_full[2],
  // grad_done[2], o_full, drain[2], dq_full, dq_free, ds_free[2], const_ready
  static constexpr int NBAR = 2 * NFIX + 2 * NSTAGE + 8 + 1 + 2 + 4 + 1;
  static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 16 + 1024;
  static constexpr int THREADS = 512;
  static constexpr int LAUNCH_REGS = 128;  // registers per thread the launch provides
  // 184 x 256 + 72 x 128 + 72 x 128 = 128 x 512
  static constexpr int EW_REGS = 184;
  static constexpr int CONTROL_REGS = 72;
  static constexpr int DRAIN_REGS = 72;
  static constexpr int LOAD_WARP = 8;
  static constexpr int SDP_WARP = 9;
  static constexpr int GRAD_WARP = 10;
  static constexpr int DRAIN_WARP0 = 12;
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_P = 256, COL_DV = 320, COL_DK = 384, COL_DQ = 448;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(DS_OFF % 1024 == 0 && STG_OFF % 1024 == 0 && ONES_OFF % 1024 == 0 && ZERO_OFF % 1024 == 0 &&
                    STAGE_BYTES % 1024 == 0,
                "swizzled buffers need 1 KB alignment");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Elementwise step of 32 query columns with the per-query terms already inside s and dp:
// P = 2^(s c2), dS = P dp, zero where `keep` is false.
template <class KEEP>
__device__ __forceinline__ void bwd64_chunk(const uint32_t* s, const uint32_t* dp, float c2, KEEP keep,
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
  uint8_t* sFix = smem + C::FIX_OFF;  // [buffer] K, V
  uint8_t* sSt = smem + C::ST_OFF;    // per stage: Q, dO, the term images
  uint8_t* sDS = smem + C::DS_OFF;    // [tile % 2] dS^T
  uint8_t* sStg = smem + C::STG_OFF;  // dQ staging
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* fix_full = bars;                // [buffer] K, V of a unit landed (units with tiles, in turn)
  uint64_t* fix_free = fix_full + C::NFIX;  // [buffer] the unit's last product reading K, V completed
  uint64_t* full = fix_free + C::NFIX;      // [stage]
  uint64_t* empty = full + C::NSTAGE;       // [stage]
  uint64_t* s_full = empty + C::NSTAGE;     // [half]: S^T and dP^T of the half are in TMEM
  uint64_t* sd_free = s_full + 2;           // [half]: ... and in the elementwise warps' registers
  uint64_t* p_full = sd_free + 2;           // [half]: P^T in TMEM and dS^T in shared memory
  uint64_t* grad_done = p_full + 2;         // [half]: the dV and dK products of the half completed
  uint64_t* o_full = grad_done + 2;         // dV and dK of a unit complete
  uint64_t* drain = o_full + 1;             // [issuer]
  uint64_t* dq_full = drain + 2;            // dQ_t is in TMEM
  uint64_t* dq_free = dq_full + 1;          // the drain warpgroup has read dQ_t
  uint64_t* ds_free = dq_free + 1;          // [buffer]: the dK and dQ products reading dS^T buffer t % 2 completed
  uint64_t* const_ready = ds_free + 2;      // the ones and zero blocks are written
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  uint32_t* ds_count = tmem_slot + 2;  // elementwise warps that have written their dS rows (8 per tile)

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int off = p.n_kv - p.n_q;  // bottom-right alignment
  const int n_qt = (p.n_q + 127) / 128;
  const int n_units = p.bh_count * ((p.n_kv + 127) / 128);
  // The k-th unit of this CTA: units are numbered heaviest first (key tile 0 of every head, then
  // key tile 1, ...), and successive rounds of gridDim.x units are dealt in alternating directions.
  auto unit_of = [&](int k) {
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    return (k & 1) ? (k + 1) * G - 1 - b : k * G + b;
  };
  struct Unit {
    int bh, j0, t_first, NT;  // query tiles t_first .. t_first + NT - 1 see some key of [j0, j0 + 128)
  };
  auto unit_at = [&](int u) {
    Unit g;
    g.bh = u % p.bh_count;
    g.j0 = (u / p.bh_count) * 128;
    g.t_first = 0;
    if (CAUSAL) {  // causal rows q with q + off >= j0
      const long long q_min = (long long)g.j0 - off;
      g.t_first = q_min <= 0 ? 0 : (int)(q_min / 128);
    }
    g.NT = g.t_first < n_qt ? n_qt - g.t_first : 0;
    return g;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NFIX; ++i) {
      mbar_init(&fix_full[i], 1);
      mbar_init(&fix_free[i], 1);
    }
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
      mbar_init(&ds_free[h], 2);  // the gradient issuer's dK and the S issuer's dQ
    }
    mbar_init(o_full, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
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
  static_assert(C::EW_REGS * 256 + C::CONTROL_REGS * 128 + C::DRAIN_REGS * 128 <= C::LAUNCH_REGS * C::THREADS,
                "register split exceeds the launch");

  const bool tmem_bad = tmem_alloc_bad(tmem);  // debug builds only
  if (tmem_bad) {
  } else if (warp >= C::DRAIN_WARP0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::DRAIN_REGS));
    // ------------------------------------------------------------ dQ drain warpgroup
    // dQ_t (TMEM lanes = the tile's queries, 64 fp32 columns), 32 columns at a time, through one
    // staging image and a TMA reduce-add into the fp32 accumulator issued by the warpgroup's first
    // thread.  The four warps agree on every drain with a barrier vote (named barrier 3), so a
    // failed wait in any of them makes all of them skip it and the later ones: each takes part in
    // exactly as many votes as the CTA has tiles, whatever fails, and none is left at a named barrier.
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const bool leader = threadIdx.x == 32 * C::DRAIN_WARP0;
    int n_votes = 0, n_tiles = 0;
    for (int k = 0, u = unit_of(0); u < n_units; u = unit_of(++k)) n_tiles += unit_at(u).NT;
    auto drain = [&](int gi, int q0, int bh, bool can) -> bool {
      const bool r = can && mbar_wait_bounded(dq_full, (uint32_t)gi & 1u, abort_flag, &timed_out);
      if (leader) bulk_wait_group_read_all();  // the previous reduces have read the staging image
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
          tma_reduce_add_3d(&tmdQacc, sStg, 32 * c, q0, bh);
          bulk_commit_group();
        }
      }
      return true;
    };
    bool ok = true;
    for (int k = 0, u = unit_of(0), g = 0; ok && u < n_units; u = unit_of(++k)) {
      const Unit U = unit_at(u);
      for (int t = 0; ok && t < U.NT; ++t) ok = drain(g + t, (U.t_first + t) * 128, U.bh, true);
      g += U.NT;
    }
    while (n_votes < n_tiles) drain(n_votes, 0, 0, false);
    if (leader) bulk_wait_group_all();  // every reduce has completed before the CTA exits
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        tma_prefetch_desc(&tmdO);
        tma_prefetch_desc(&tmdQacc);
        int issued = 0, nf = 0;  // ring indices issued, units whose K, V were loaded
        bool ok = true;
        for (int k = 0, u = unit_of(0), g = 0; ok && u < n_units; u = unit_of(++k)) {
          const Unit U = unit_at(u);
          if (U.NT == 0) continue;
          // K, V replace those of the unit NFIX units back once its last S^T, dP^T and dQ products have run
          const int b = nf % C::NFIX;
          if (nf >= C::NFIX &&
              !(ok = mbar_wait_bounded(&fix_free[b], (uint32_t)(nf / C::NFIX - 1) & 1u, abort_flag, &timed_out)))
            break;
          mbar_arrive_expect_tx(&fix_full[b], 2 * C::TILE_BYTES);
          tma_load_3d(sFix + b * 2 * C::TILE_BYTES, &tmK, &fix_full[b], 0, U.j0, U.bh);
          tma_load_3d(sFix + b * 2 * C::TILE_BYTES + C::TILE_BYTES, &tmV, &fix_full[b], 0, U.j0, U.bh);
          ++nf;
          for (int t = 0; t < U.NT; ++t) {
            const int gi = g + t, st = gi % C::NSTAGE;
            if (!(ok = mbar_wait_bounded(&empty[st], ((uint32_t)(gi / C::NSTAGE) & 1u) ^ 1u, abort_flag, &timed_out)))
              break;
            uint8_t* dst = sSt + st * C::STAGE_BYTES;
            const int qt = U.t_first + t;
            mbar_arrive_expect_tx(&full[st], 2 * C::TILE_BYTES + C::TERM_BYTES);
            tma_load_3d(dst, &tmQ, &full[st], 0, qt * 128, U.bh);
            tma_load_3d(dst + C::TILE_BYTES, &tmdO, &full[st], 0, qt * 128, U.bh);
            bulk_load(dst + 2 * C::TILE_BYTES, p.aug + ((size_t)U.bh * (p.n_q_pad / 128) + qt) * C::TERM_BYTES,
                      C::TERM_BYTES, &full[st]);
            issued = gi + 1;
          }
          g += U.NT;
        }
        if (*abort_flag) {  // let the copies in flight land before the CTA exits
          for (int i = (nf > C::NFIX ? nf - C::NFIX : 0); i < nf; ++i)
            mbar_wait_drain(&fix_full[i % C::NFIX], (uint32_t)(i / C::NFIX) & 1u);
          for (int gi = (issued > C::NSTAGE ? issued - C::NSTAGE : 0); gi < issued; ++gi)
            mbar_wait_drain(&full[gi % C::NSTAGE], (uint32_t)(gi / C::NSTAGE) & 1u);
        }
      }
    } else if (warp == C::SDP_WARP || warp == C::GRAD_WARP) {
      // ------------------------------------------------------------ MMA issuers
      const int role = warp - C::SDP_WARP;  // 0: S^T, dP^T and dQ; 1: dV and dK
      if (lane == 0) {
        auto wait_bar = [&](uint64_t* bar, int phase) {
          const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
          if (r) tc_fence_after_sync();  // the elementwise warps' TMEM and shared-memory writes precede the products
          return r;
        };
        const uint32_t fix = smem_u32(sFix), st0 = smem_u32(sSt), ds0 = smem_u32(sDS);
        bool ok = true;
        if (role == 0) {
          // S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = the tile's 128 queries, K = d): K, V and
          // the stage's Q, dO rows all K-major; then the term step: A = the ones block (M = 128 keys
          // in two 64-key images 1 KB apart, MN-major), B = the tile's term images (N = queries,
          // MN-major), rows 8-15 of both read the zeros.
          constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false), idT = idesc_bf16_f32(128, 128, true, true);
          uint64_t dK = 0, dV = 0, dKm = 0;  // this unit's K, V buffer (set per unit)
          const uint32_t ones = smem_u32(smem + C::ONES_OFF), zero = smem_u32(smem + C::ZERO_OFF);
          const uint64_t dOnes = smem_desc_sw128(ones, 1024, zero - ones);
          // dQ_t = dS_t K (M = 128 queries, N = d, K = 128 keys): dS read MN-major from dS buffer
          // t % 2 (two 64-query blocks 16 KB apart), K MN-major like V in the forward.
          constexpr uint32_t idQ = idesc_bf16_f32(128, 64, true, true);
          // dQ_gi may be formed once both halves' dS_gi are in shared memory (eight elementwise
          // warps per tile: a count, since this issuer reads it up to a tile late) and dQ_(gi-1)
          // has left TMEM
          auto issue_dq = [&](int gi) {
            bool r = count_wait_bounded(ds_count, 8u * (uint32_t)(gi + 1), abort_flag, &timed_out);
            if (r) tc_fence_after_sync();
            if (r && gi > 0) r = wait_bar(dq_free, gi - 1);
            if (!r) return false;
            const uint64_t dSm = smem_desc_sw128(ds0 + (uint32_t)((gi & 1) * C::DS_BYTES), C::TILE_BYTES, 1024);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t o = (uint64_t)((kk * 2048) >> 4);  // 16 keys
              mma_ss(tmem + C::COL_DQ, dSm + o, dKm + o, idQ, kk > 0 ? 1u : 0u);
            }
            tc_commit(dq_full);
            tc_commit(&ds_free[gi & 1]);
            return true;
          };
          ok = wait_bar(const_ready, 0);
          for (int k = 0, u = unit_of(0), g = 0, nf = 0; ok && u < n_units; u = unit_of(++k)) {
            const Unit U = unit_at(u);
            if (U.NT == 0) continue;
            const int b = nf % C::NFIX;
            if (!(ok = wait_bar(&fix_full[b], nf / C::NFIX))) break;
            const uint32_t kv = fix + (uint32_t)(b * 2 * C::TILE_BYTES);
            dK = smem_desc_sw128(kv, 16, 1024);
            dV = smem_desc_sw128(kv + C::TILE_BYTES, 16, 1024);
            dKm = smem_desc_sw128(kv, C::TILE_BYTES, 1024);
            for (int t = 0; ok && t < U.NT; ++t) {
              const int gi = g + t, st = gi % C::NSTAGE;
              if (!(ok = wait_bar(&full[st], gi / C::NSTAGE))) break;
              // both halves of the previous tile (this unit's or the last one's) are in registers
              if (gi > 0 && !(ok = wait_bar(&sd_free[0], gi - 1) && wait_bar(&sd_free[1], gi - 1))) break;
              const uint32_t sq = st0 + st * C::STAGE_BYTES;
              const uint64_t dQk = smem_desc_sw128(sq, 16, 1024), dOk = smem_desc_sw128(sq + C::TILE_BYTES, 16, 1024);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                const uint64_t o = (uint64_t)((kk * 32) >> 4);
                mma_ss(tmem + C::COL_S, dK + o, dQk + o, idS, kk > 0 ? 1u : 0u);
                mma_ss(tmem + C::COL_DP, dV + o, dOk + o, idS, kk > 0 ? 1u : 0u);
              }
              const uint32_t img = sq + 2 * C::TILE_BYTES;  // images [S h0, S h1, dP h0, dP h1]
              mma_ss(tmem + C::COL_S, dOnes, smem_desc_sw128(img, 1024, zero - img), idT, 1u);
              mma_ss(tmem + C::COL_DP, dOnes, smem_desc_sw128(img + 2048, 1024, zero - img - 2048), idT, 1u);
              tc_commit(&s_full[0]);
              tc_commit(&s_full[1]);
              if (t > 0 && !(ok = issue_dq(gi - 1))) break;  // the previous tile of this unit
            }
            // the unit's last dQ, then K and V may be replaced
            if (!ok || !(ok = issue_dq(g + U.NT - 1))) break;
            tc_commit(&fix_free[b]);
            g += U.NT;
            ++nf;
          }
        } else {
          // dV += P^T_h dO_h (A = P^T from TMEM), dK += dS^T_h Q_h (A = dS^T K-major from shared
          // memory), M = 128 keys, N = d, K = the 64 queries of half h; dO_h, Q_h MN-major.  A unit's
          // first products overwrite the accumulators: its first P^T only arrives after the
          // elementwise warps have read the previous unit's dV, dK out.
          constexpr uint32_t idG = idesc_bf16_f32(128, 64, false, true);
          for (int k = 0, u = unit_of(0), g = 0; ok && u < n_units; u = unit_of(++k)) {
            const Unit U = unit_at(u);
            if (U.NT == 0) continue;
            for (int t = 0; ok && t < U.NT; ++t) {
              const int gi = g + t, st = gi % C::NSTAGE;
              const uint32_t sq = st0 + st * C::STAGE_BYTES;
              const uint64_t dQm = smem_desc_sw128(sq, C::TILE_BYTES, 1024), dOm = smem_desc_sw128(sq + C::TILE_BYTES, C::TILE_BYTES, 1024);
              const uint32_t dsb = ds0 + (uint32_t)((gi & 1) * C::DS_BYTES);
              for (int h = 0; ok && h < 2; ++h) {
                if (!(ok = wait_bar(&p_full[h], gi))) break;
                // a unit's first products overwrite dV (read out by warpgroup 0) and dK (by warpgroup
                // 1): both warpgroups must have handed in the unit's first tile
                if (t == 0 && h == 0 && !(ok = wait_bar(&p_full[1], gi))) break;
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
                  tc_commit(&ds_free[gi & 1]);  // with the S issuer's commit after dQ_gi
                }
              }
            }
            if (ok) tc_commit(o_full);  // the unit's dV, dK
            g += U.NT;
          }
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
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const float c2 = p.scale_log2;
    bool ok = true;
    auto wait_warp = [&](uint64_t* bar, int phase) {
      const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      return __all_sync(0xffffffffu, r);
    };
    {  // the ones block (rows 0-2 of both 64-key images) and the zeros, 16 bytes per thread
      const int i = threadIdx.x;  // 0 .. 255
      const uint32_t one2 = 0x3F803F80u;  // two bf16 ones
      const bool ones_row = i < 128 && ((i & 63) >> 3) < 3;  // byte (i & 63) * 16 of image i >> 6: row (i & 63) / 8
      *reinterpret_cast<uint4*>(smem + C::ONES_OFF + i * 16) =
          ones_row ? make_uint4(one2, one2, one2, one2) : make_uint4(0u, 0u, 0u, 0u);
      if (i >= 128) *reinterpret_cast<uint4*>(smem + C::ZERO_OFF + (i - 128) * 16) = make_uint4(0u, 0u, 0u, 0u);
      fence_proxy_async_smem();
      mbar_arrive(const_ready);
    }
    for (int k = 0, u = unit_of(0), g = 0, nf = 0; ok && u < n_units; u = unit_of(++k)) {
      const Unit U = unit_at(u);
      const int key = U.j0 + row;
      for (int t = 0; ok && t < U.NT; ++t) {
        const int gi = g + t;
        if (!(ok = wait_warp(&s_full[w], gi))) break;
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
        mbar_arrive(&sd_free[w]);  // the next S^T, dP^T may be formed
        // P^T columns: read by the dV product of the previous tile; dS^T buffer gi % 2: read by the
        // dK and dQ products of tile gi - 2
        if (gi > 0 && !(ok = wait_warp(&grad_done[w], gi - 1))) break;
        if (gi > 1 && !(ok = wait_warp(&ds_free[gi & 1], gi / 2 - 1))) break;
        tc_fence_after_sync();
        const int q0 = (U.t_first + t) * 128 + 64 * w;  // first query of this warpgroup's columns
        const bool masked = CAUSAL && (q0 + off < U.j0 + 127);
        uint8_t* drow = sDS + (gi & 1) * C::DS_BYTES + w * C::TILE_BYTES + (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pp[16], ps[16];
          const int qc = q0 + 32 * h;
          if (masked)
            bwd64_chunk(s + 32 * h, dp + 32 * h, c2, [&](int c) { return key <= qc + c + off; }, pp, ps);
          else
            bwd64_chunk(s + 32 * h, dp + 32 * h, c2, [&](int) { return true; }, pp, ps);
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
        __syncwarp();
        if (lane == 0) red_release_add(ds_count, 1u);
      }
      // ------------------------------------------------------------ the unit's epilogue
      if (ok && U.NT > 0) ok = wait_warp(o_full, nf);
      if (ok) {
        tc_fence_after_sync();
        // warpgroup 0 writes dV, warpgroup 1 writes dK (times scale); zeros if no query sees the tile
        const uint32_t col = w ? C::COL_DK : C::COL_DV;
        const float mul = w ? p.scale : 1.f;
        const bool store = key < p.n_kv;
        __nv_bfloat16* dst = (w ? p.dK : p.dV) + ((size_t)U.bh * p.n_kv + (store ? key : 0)) * C::D;
#pragma unroll 1
        for (int cb = 0; cb < C::D; cb += 32) {
          uint32_t o[32];
          if (U.NT > 0) {
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
        tc_fence_before_sync();  // dV, dK read out before the next unit's first products (after its first P^T)
      }
      if (U.NT > 0) ++nf;
      g += U.NT;
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
