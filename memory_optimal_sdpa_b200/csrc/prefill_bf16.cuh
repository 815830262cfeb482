// prefill_bf16.cuh -- exact SDPA forward, bf16 in / bf16 out, on the sm_100a tensor cores.
//
// The memory-optimal form of attention (MoA paper abstract, "Attention at the
// Theoretical Minimum"; agents-report.net MoA article, "DNF derivation"): every
// intermediate array -- the score matrix, the probabilities and the transposed
// keys -- lives only in on-chip memory (TMEM, registers, shared memory), so the
// kernel reads Q, K and V and writes O and LSE exactly once: O(n*d_k + n*d_v)
// global traffic.  The index space is lifted onto the B200 hierarchy as
// 128-row tiles: one work unit is one (batch, head) and two adjacent 128-row
// query tiles (a, b), streamed against 128-row key/value tiles.
//
// Warp roles (384 threads, three warpgroups):
//   warps 0-3  softmax warpgroup for query tile a (thread t owns TMEM lane = row t)
//   warps 4-7  softmax warpgroup for query tile b
//   warp  8    TMA producer: Q once, then K_j, V_j into a ring of shared-memory slots
//   warp  9    MMA issuer for query tile a (one thread) and TMEM owner
//   warp  10   MMA issuer for query tile b (one thread)
//   warp  11   idle
// Registers: each SM sub-partition holds 16K 32-bit registers and receives
// one warp of every warpgroup, so the CTA launches at 168 per thread and then
// moves registers from the producer/MMA warpgroup to the two softmax
// warpgroups: d = 64 72 and 216 (2*216 + 72 <= 512 per sub-partition lane slot,
// 72*128 + 216*256 = 384*168 in total), d = 128 88 and 208 (the same totals),
// where the MMA issuers' shared-S bookkeeping spills at 72 and the softmax
// still fits in 208 (measured: 1 x 32 x 8192 with a 512-key window 533 -> 561
// TF/s, the others unchanged or within noise; at d = 64 the 216 pays, by 1 %).
//
// TMEM (512 columns).  d = 64: S_a [0,128), S_b [128,256), P_a [256,320),
// P_b [320,384), O_a [384,448), O_b [448,512).  With P in its own columns the
// softmax releases S_x as soon as it has loaded it, so the tensor core computes
// S_x(j+1) while the softmax of tile j still runs.  d = 128: two S tiles and two
// O tiles would fill the memory and leave P only the columns of its own S (then
// the next S waits for P V), so instead one S buffer [0,128) serves both query
// tiles in turn -- S_a(j), S_b(j), S_a(j+1), ..., each product issued once every
// earlier one has been read into registers (a count in shared memory) -- and
// P_a [128,192), P_b [192,256), O_a [256,384), O_b [384,512).  Measured against
// P over S: 1 x 8 x 32768 full 1044 -> 1160 TF/s, 1 x 32 x 8192 causal 1048 -> 1166.
//
// The online softmax keeps, per row, the running maximum m (in log2 units of
// the scaled logits) and sum l; O and l are rescaled only when m grows by more
// than 8 (a factor 256): O and l always share the same reference maximum, so
// O/l is exact whatever reference is used, and fp32 cannot overflow.  At d = 64,
// on tiles without masked entries, one column pair in eight takes its
// exponentials on the FMA pipe (sm100::exp2_poly2) instead of the MUFU unit
// (measured: cfg2 537 -> 551 TF/s; at d = 128 it does not pay).
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

#ifndef SDPA_SHARED_S_D128
#define SDPA_SHARED_S_D128 1  // d = 128: one S buffer taken in turn by both query tiles, P in its own columns
#endif
#ifndef SDPA_EXP2_POLY_EVERY_D64
#define SDPA_EXP2_POLY_EVERY_D64 8  // every 8th column pair of an unmasked tile on the FMA pipe at d = 64
#endif
#ifndef SDPA_EXP2_POLY_EVERY_D128
#define SDPA_EXP2_POLY_EVERY_D128 0  // the same at d = 128 (0: all exponentials on the MUFU unit)
#endif

namespace sdpa {

template <int D>
struct PrefillCfg {
  static constexpr int TILE_BYTES = 128 * D * 2;        // one 128 x D bf16 tile
  static constexpr int BLOCK_BYTES = 128 * 64 * 2;      // one 128-row x 64-column swizzle block (16 KB)
  static constexpr int NSLOT = (D == 128) ? 4 : 8;      // K/V ring slots
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
  // q_full, full[NSLOT], empty[NSLOT], s_full[2], s_free[2], p_full[2], pv_done[2], o_full[2], drain[2], turn[8],
  // q_free, o_free[2]
  static constexpr int NBAR = 1 + 2 * NSLOT + 2 * 6 + 8 + 3;
  // + tmem slot, abort flag, eight debug counters, the shared-S load count, align slack
  static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 48 + 1024;
  static_assert(4 + 4 + 8 * 4 + 4 <= 48, "words after the barriers");
  static constexpr int THREADS = 384;
  static constexpr int SOFTMAX_REGS = (D == 128) ? 208 : 216;
  static constexpr int CONTROL_REGS = (D == 128) ? 88 : 72;
  static constexpr int LOAD_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr uint32_t TMEM_COLS = 512;
  // d = 128: S, O of two tiles would fill the 512 columns, leaving P nowhere but over S.  Instead
  // the two tiles take turns on one S buffer (S_a(j), S_b(j), S_a(j+1), ... each issued once the
  // one before it in that order is in its softmax's registers), so P_x gets columns of its own and
  // the next S no longer waits for P_x V.
  static constexpr bool SHARED_S = (D == 128) && SDPA_SHARED_S_D128;
  static constexpr bool P_SEPARATE = (D == 64) || SHARED_S;
  static constexpr int POLY_EVERY = (D == 64) ? SDPA_EXP2_POLY_EVERY_D64 : SDPA_EXP2_POLY_EVERY_D128;  // FMA-pipe exps
  __host__ __device__ static constexpr uint32_t col_s(int x) { return SHARED_S ? 0u : (uint32_t)x * 128u; }
  __host__ __device__ static constexpr uint32_t col_p(int x) {
    return D == 64 ? 256u + (uint32_t)x * 64u : (SHARED_S ? 128u + (uint32_t)x * 64u : col_s(x));
  }
  __host__ __device__ static constexpr uint32_t col_o(int x) {
    return D == 64 ? 384u + (uint32_t)x * 64u : 256u + (uint32_t)x * 128u;
  }
};

__device__ int g_sdpa_error;  // first device-side error since the last read (0 = none)

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_sdpa_error, 0, code); }

// Debug builds (-DSDPA_DEBUG=1) add device-side consistency checks, the stand-in for a race
// checker on this hardware; a failed check records SDPA_ERR_DEVICE_CHECK (8).  Every tensor-core
// kernel here runs one CTA per SM and allocates TMEM from column 0, so its allocation must come
// back at lane 0, column 0; if it does not, the CTA does no work.
#ifndef SDPA_DEBUG
#define SDPA_DEBUG 0
#endif
__device__ __forceinline__ bool tmem_alloc_bad(uint32_t tmem) {
#if SDPA_DEBUG
  if (tmem != 0u) {
    if (threadIdx.x == 0) record_error(8 /* SDPA_ERR_DEVICE_CHECK */);
    return true;
  }
#endif
  (void)tmem;
  return false;
}

struct PrefillParams {
  __nv_bfloat16* O;
  float* LSE;
  int n_q, n_kv, bh_count, n_pairs;
  // Units are numbered group of heads by group of heads: within a group of `heads_per_group`
  // (batch, head) slices (the last group may hold fewer), heaviest query-tile pair first and
  // the group's heads side by side.  CTAs running at the same time then stream the keys and
  // values of few heads, which stay in L2 for all of them.
  int heads_per_group;
  float scale_log2;  // |scale| * log2(e), > 0 (2^-126 stands for scale = 0)
  // scale < 0: the S product is issued with A negated (S = -Q K^T), so the kernel always
  // works with a non-negative factor |scale| (the instruction descriptor's negate-A bit).
  int negate_s;
  // Local window (mask mode 2 only): query row i (key position p = i + n_kv - n_q)
  // sees keys p - win_left <= j <= p + win_right; -1 leaves a side open.
  int win_left, win_right;
};

// Key tiles [first, first + count) that query tile [r0, r0 + 128) must visit.
__host__ __device__ inline void prefill_kv_range(int r0, int n_q, int n_kv, int win_left, int win_right,
                                                 int* first, int* count) {
  *first = 0;
  *count = 0;
  if (r0 >= n_q) return;
  const int last_row = (r0 + 127 < n_q - 1) ? r0 + 127 : n_q - 1;
  const long long off = (long long)n_kv - n_q;  // bottom-right alignment
  long long hi = n_kv - 1, lo = 0;
  if (win_right >= 0 && last_row + off + win_right < hi) hi = last_row + off + win_right;
  if (win_left >= 0 && r0 + off - win_left > lo) lo = r0 + off - win_left;
  if (hi < lo) return;
  *first = (int)(lo / 128);
  *count = (int)(hi / 128) - *first + 1;
}

// Heads per unit group (see PrefillParams::heads_per_group).  Full attention: every unit weighs
// the same, so one head at a time (the CTAs of a round share one or two heads' keys and values).
// Causal or windowed: unit weights fall with the pair index, and only the order "heaviest pair
// of every head first" lets the alternating deal balance the CTAs (simulated max/mean load on a
// 1 x 32 x 8192 causal call: 1.02 with all heads in one group, 1.15-1.47 with groups of 1-16
// heads), so all heads form one group and keys are re-read from DRAM instead.
__host__ __device__ inline int prefill_heads_per_group(int mask, int bh_count) { return mask == 0 ? 1 : bh_count; }

#ifndef SDPA_SM_INTPACK
#define SDPA_SM_INTPACK 0
#endif
#ifndef SDPA_SM_TURN
#define SDPA_SM_TURN 1
#endif
#ifndef SDPA_SM_TURN_WARP
#define SDPA_SM_TURN_WARP 1
#endif
#ifndef SDPA_SM_TURN_NAMED
#define SDPA_SM_TURN_NAMED 1  // pass the turn with hardware named barriers (else mbarriers)
#endif

// Two finite, non-negative floats -> bf16x2 (lo in bits 0..15), rounded to nearest.
// Default: the packed conversion instruction (measured on B200 at 62 per clock per SM, on a
// unit of its own beside the 16 per clock of ex2).  SDPA_SM_INTPACK=1 rounds with integer adds
// and a byte permute instead (ties away from zero; 29 per clock per SM), measured no faster.
__device__ __forceinline__ uint32_t pack_p(float lo, float hi) {
#if SDPA_SM_INTPACK
  return __byte_perm(__float_as_uint(lo) + 0x8000u, __float_as_uint(hi) + 0x8000u, 0x7632);
#else
  return sm100::pack_bf16x2(lo, hi);
#endif
}

// Exponentials of one 128-score row: p = 2^(s*c2 - m), bf16 pairs into pk, returns sum p.
// EVERY > 0: every EVERY-th pair on the FMA pipe (finite scores only).
template <int EVERY>
__device__ __forceinline__ float softmax_exp_row(const uint32_t (&s)[128], float c2, float m_use, uint32_t (&pk)[64]) {
  using namespace sm100;
  const float2 cc = make_float2(c2, c2), nm = make_float2(-m_use, -m_use);
  float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float2 xv = ffma2(make_float2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])), cc, nm);
    float2 e;
    if (EVERY > 0 && (i % (EVERY > 0 ? EVERY : 1)) == EVERY - 1) {
      e = exp2_poly2(xv);
    } else {
      e.x = ex2_approx(xv.x);
      e.y = ex2_approx(xv.y);
    }
    if (i & 1)
      acc1 = fadd2(acc1, e);
    else
      acc0 = fadd2(acc0, e);
    pk[i] = pack_p(e.x, e.y);
  }
  const float2 a = fadd2(acc0, acc1);
  return a.x + a.y;
}

// MASK: 0 full attention, 1 causal (bottom-right aligned), 2 local window (p.win_left, p.win_right).
// Modes 0 and 1 fix the bounds at compile time, so their key ranges and masks fold to constants.
//
// Persistent: each CTA takes work units (one (batch, head) and two adjacent query tiles) from
// the unit list, heaviest first, dealt round by round in alternating directions.  TMEM, barriers and descriptor prefetches
// are set up once; every barrier's phase runs on across units (counters of ring slots, rounds
// and units per role), and the next unit's Q, K, V loads and first S products proceed while
// the softmax warpgroups still write the previous unit's output.  Two barriers guard what a
// unit hands to the next: q_free (both issuers' last S of the unit has run: Q may be
// replaced) and o_free[x] (the epilogue has read O_x: the next P_x V may overwrite it).
template <int D, int MASK>
__global__ void __launch_bounds__(384, 1)
    sdpa_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using C = PrefillCfg<D>;
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sKV = smem + C::KV_OFF;
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + C::NSLOT;
  uint64_t* s_full = empty + C::NSLOT;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* o_full = pv_done + 2;
  uint64_t* drain = o_full + 2;
  uint64_t* turn = drain + 2;      // [query tile][warp within the warpgroup]
  uint64_t* q_free = turn + 8;     // both issuers' S products of a unit have run
  uint64_t* o_free = q_free + 1;   // [query tile]: the epilogue has read O_x
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  // debug builds: final counters of each role, for the barrier-phase check at teardown
  // [0] units loaded, [1] ring indices loaded, [2 + x] rounds of tile x, [4 + x] units with rounds
  // of tile x (softmax x), [6 + x] units seen by issuer x
  int* dbg = (int*)(tmem_slot + 2);
  // shared S buffer (d = 128): warps that have read an S product into registers, 4 per product
  uint32_t* s_loads = tmem_slot + 10;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_units = p.bh_count * p.n_pairs;
  const int win_left = MASK == 2 ? p.win_left : -1;
  const int win_right = MASK == 2 ? p.win_right : (MASK == 1 ? 0 : -1);

  // The k-th unit of this CTA: units are numbered heaviest first, and successive rounds of
  // gridDim.x units are dealt in alternating directions, so a CTA that takes a heavy unit in one
  // round takes a light one in the next (balanced totals under a causal mask).
  auto unit_of = [&](int k) {
    const int G = (int)gridDim.x, b = (int)blockIdx.x;
    return (k & 1) ? (k + 1) * G - 1 - b : k * G + b;
  };
  // Geometry of work unit u: heaviest query-tile pairs (the last rows, under a causal mask) first.
  struct Unit {
    int bh, r0a, r0b, fa, ta, fb, tb, T, J0, TL;
  };
  auto unit_at = [&](int u) {
    Unit g;
    const int per_group = p.heads_per_group * p.n_pairs;  // units of a full group
    const int grp = u / per_group;
    const int r = u - grp * per_group;
    const int h0 = grp * p.heads_per_group;
    const int hg = (p.bh_count - h0 < p.heads_per_group) ? p.bh_count - h0 : p.heads_per_group;
    g.bh = h0 + r % hg;
    const int pair = p.n_pairs - 1 - r / hg;
    g.r0a = pair * 256;
    g.r0b = g.r0a + 128;
    prefill_kv_range(g.r0a, p.n_q, p.n_kv, win_left, win_right, &g.fa, &g.ta);  // first key tile, count
    prefill_kv_range(g.r0b, p.n_q, p.n_kv, win_left, win_right, &g.fb, &g.tb);
    g.T = g.ta > g.tb ? g.ta : g.tb;  // softmax rounds
    // Key tiles loaded: J0 .. J0 + TL - 1, the union of both ranges.
    const int J1 = g.ta == 0 ? g.fb + g.tb - 1
                             : (g.tb == 0 ? g.fa + g.ta - 1 : (g.fa + g.ta > g.fb + g.tb ? g.fa + g.ta - 1 : g.fb + g.tb - 1));
    g.J0 = g.ta == 0 ? g.fb : (g.tb == 0 ? g.fa : (g.fa < g.fb ? g.fa : g.fb));
    g.TL = (g.ta == 0 && g.tb == 0) ? 0 : J1 - g.J0 + 1;
    return g;
  };

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 2);  // released by both MMA issuers
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&s_free[x], 128);
      mbar_init(&p_full[x], 128);
      mbar_init(&pv_done[x], 1);
      mbar_init(&o_full[x], 1);
      mbar_init(&o_free[x], 128);
    }
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    mbar_init(q_free, 2);
    for (int w = 0; w < 8; ++w) mbar_init(&turn[w], SDPA_SM_TURN_WARP ? 32 : 128);
    *abort_flag = 0;
    *s_loads = 0;
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
  static_assert(C::SOFTMAX_REGS * 256 + C::CONTROL_REGS * 128 <= 168 * 384, "register split exceeds the launch");
  const bool tmem_bad = tmem_alloc_bad(tmem);

  if (tmem_bad) {
  } else if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        int ring = 0, nu = 0, issued = 0;  // ring base of this unit, units whose Q was loaded, ring indices issued
        bool ok = true;
        for (int k = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++k)) {
          const Unit g = unit_at(u);
          // Q of this unit replaces the previous unit's once both issuers' S products of it have run.
          if (nu > 0 && !(ok = mbar_wait_bounded(q_free, (uint32_t)(nu - 1) & 1u, abort_flag, &timed_out))) break;
          mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
              tma_load_3d(sQ + x * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmQ, q_full, cb * 64, x ? g.r0b : g.r0a, g.bh);
          ++nu;
          for (int idx = 0; idx < 2 * g.TL; ++idx) {
            const int gi = ring + idx;
            const int slot = gi % C::NSLOT;
            if (!(ok = mbar_wait_bounded(&empty[slot], ((uint32_t)(gi / C::NSLOT) & 1u) ^ 1u, abort_flag, &timed_out)))
              break;
            mbar_arrive_expect_tx(&full[slot], C::TILE_BYTES);
            const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
            uint8_t* dst = sKV + slot * C::TILE_BYTES;
#pragma unroll
            for (int cb = 0; cb < D / 64; ++cb)
              tma_load_3d(dst + cb * C::BLOCK_BYTES, map, &full[slot], cb * 64, (g.J0 + (idx >> 1)) * 128, g.bh);
            issued = gi + 1;
          }
          if (!ok) break;
          ring += 2 * g.TL;
        }
        if (SDPA_DEBUG) dbg[0] = nu, dbg[1] = ring;
        if (*abort_flag) {  // let the copies already in flight land before the CTA exits
          if (nu > 0) mbar_wait_drain(q_full, (uint32_t)(nu - 1) & 1u);
          for (int gi = (issued > C::NSLOT ? issued - C::NSLOT : 0); gi < issued; ++gi)
            mbar_wait_drain(&full[gi % C::NSLOT], (uint32_t)(gi / C::NSLOT) & 1u);
        }
      }
    } else if (warp == C::MMA_WARP || warp == C::MMA_WARP + 1) {
      // ------------------------------------------------------------ MMA issuers
      // Query tile x's MMAs are issued by lane 0 of warp MMA_WARP + x, so the two
      // instruction streams (and their barrier waits) proceed in parallel.  Within one
      // stream tcgen05 MMAs execute in issue order, which is what lets P_x alias S_x when
      // P has no columns of its own.
      const int x = warp - C::MMA_WARP;
      if (lane == 0) {
        // Q (K-major) x K (K-major); bit 13 negates A (Q) for a negative scale
        const uint32_t idS = idesc_bf16_f32(128, 128, false, false) | (p.negate_s ? (1u << 13) : 0u);
        constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);     // P (TMEM) x V (MN-major)
        const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);
        // Descriptors are built once; every operand tile is then reached by adding its byte
        // offset >> 4 to the start-address field (the low 14 bits; shared memory < 256 KB, so
        // the add never carries out of the field).
        const uint64_t dQ = smem_desc_sw128(sQa + x * C::TILE_BYTES, 16, 1024);  // K-major
        const uint64_t dK = smem_desc_sw128(sKVa, 16, 1024);                     // K-major
        const uint64_t dV = smem_desc_sw128(sKVa, C::BLOCK_BYTES, 1024);         // MN-major
        const uint32_t tS = tmem + C::col_s(x), tP = tmem + C::col_p(x), tO = tmem + C::col_o(x);
        auto wait_bar = [&](uint64_t* bar, int phase) {
          const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
          if (r) tc_fence_after_sync();
          return r;
        };
        auto wait_slot = [&](int gi) { return wait_bar(&full[gi % C::NSLOT], gi / C::NSLOT); };
        // running counts: ring indices of earlier units, units, rounds of tile x, units with rounds,
        // S products of both tiles in earlier units (the shared S buffer's order)
        int ring = 0, nu = 0, rx = 0, ox = 0, sbase = 0;
        bool ok = true;
        for (int k = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++k)) {
          const Unit g = unit_at(u);
          const int tx = x ? g.tb : g.ta;
          const int lead = tx ? (x ? g.fb : g.fa) - g.J0 : g.TL;  // loaded key tiles before this tile's first
          const int k0 = ring + 2 * lead;                         // ring index of this tile's first K
          // r: this query tile's r-th key tile
          auto issue_S = [&](int r) {  // S_x = Q_x K^T
            const uint64_t b0 = dK + (uint64_t)((((k0 + 2 * r) % C::NSLOT) * C::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = (uint64_t)((((kk >> 2) * C::BLOCK_BYTES) + (kk & 3) * 32) >> 4);
              mma_ss(tS, dQ + off, b0 + off, idS, kk > 0 ? 1u : 0u);
            }
          };
          auto issue_PV = [&](int r) {  // O_x += P_x V
            const uint64_t b0 = dV + (uint64_t)((((k0 + 2 * r + 1) % C::NSLOT) * C::TILE_BYTES) >> 4);
#pragma unroll
            for (int kk = 0; kk < 128 / 16; ++kk)
              mma_ts(tO, tP + kk * 8, b0 + (uint64_t)((kk * 2048) >> 4), idO, (r > 0 || kk > 0) ? 1u : 0u);
          };
          // Shared S buffer: S_x(r) is the seq-th product in the order S_a(0), S_b(0), S_a(1), ...
          // (tiles without a round r skipped) and may be issued once every product before it has
          // been read into registers (4 warps each).  A count, not a barrier phase: an issuer
          // whose tile has no round left can run a unit ahead of the other one.
          auto wait_s_turn = [&](int r) {
            const int seq = sbase + (x == 0 ? r + (r < g.tb ? r : g.tb) : (r + 1 < g.ta ? r + 1 : g.ta) + r);
            const bool ready = count_wait_bounded(s_loads, 4u * (uint32_t)seq, abort_flag, &timed_out);
            if (ready) tc_fence_after_sync();
            return ready;
          };
          if (!(ok = wait_bar(q_full, nu))) break;
          // Key tiles only the other query tile uses are released, in order, once they have landed.
          for (int gi = ring; ok && gi < k0; ++gi) {
            if (!(ok = wait_slot(gi))) break;
            mbar_arrive(&empty[gi % C::NSLOT]);
          }
          if (ok && tx > 0) {
            // S_x is free once the softmax has read the previous unit's last S_x (with P aliasing
            // S_x, the previous P_x V was issued first on this stream)
            if (C::SHARED_S) ok = wait_s_turn(0);
            else if (C::P_SEPARATE && rx > 0) ok = wait_bar(&s_free[x], rx - 1);
            if (ok && (ok = wait_slot(k0))) {
              issue_S(0);
              tc_commit(&s_full[x]);
              tc_commit(&empty[k0 % C::NSLOT]);
            }
          }
          if (ok && tx <= 1) tc_commit(q_free);  // this unit's S products of tile x are all issued
          for (int j = 0; ok && j < tx; ++j) {
            if (C::P_SEPARATE && j + 1 < tx) {
              // next S as soon as the softmax has read the current one
              if (!(ok = wait_slot(k0 + 2 * (j + 1)) &&
                         (C::SHARED_S ? wait_s_turn(j + 1) : wait_bar(&s_free[x], rx + j))))
                break;
              issue_S(j + 1);
              tc_commit(&s_full[x]);
              tc_commit(&empty[(k0 + 2 * (j + 1)) % C::NSLOT]);
              if (j + 2 == tx) tc_commit(q_free);
            }
            if (!(ok = wait_slot(k0 + 2 * j + 1) && wait_bar(&p_full[x], rx + j))) break;  // V and P_x of tile j
            if (j == 0 && ox > 0 && !(ok = wait_bar(&o_free[x], ox - 1))) break;  // O_x read by the last epilogue
            issue_PV(j);
            if (C::P_SEPARATE) tc_commit(&pv_done[x]);
            if (j == tx - 1) tc_commit(&o_full[x]);
            tc_commit(&empty[(k0 + 2 * j + 1) % C::NSLOT]);
            if (!C::P_SEPARATE && j + 1 < tx) {
              // P_x aliases S_x: the next S_x is issued after P_x V (same stream, in order)
              if (!(ok = wait_slot(k0 + 2 * (j + 1)))) break;
              issue_S(j + 1);
              tc_commit(&s_full[x]);
              tc_commit(&empty[(k0 + 2 * (j + 1)) % C::NSLOT]);
              if (j + 2 == tx) tc_commit(q_free);
            }
          }
          for (int gi = k0 + 2 * tx; ok && gi < ring + 2 * g.TL; ++gi) {
            if (!(ok = wait_slot(gi))) break;
            mbar_arrive(&empty[gi % C::NSLOT]);
          }
          ring += 2 * g.TL;
          ++nu;
          rx += tx;
          sbase += g.ta + g.tb;
          if (tx > 0) ++ox;
        }
        if (SDPA_DEBUG) dbg[6 + x] = nu;
        // Every MMA and every commit issued above has landed before TMEM is released
        // and before the CTA's shared memory (which the commits arrive on) goes away.
        tc_commit(&drain[x]);
        mbar_wait_drain(&drain[x], 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
    // ------------------------------------------------ softmax + epilogue warpgroups
    const int x = warp >> 2;  // query tile a (0) or b (1)
    const int t = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + C::col_s(x) + lane_base;
    const uint32_t tP = tmem + C::col_p(x) + lane_base;
    const uint32_t tO = tmem + C::col_o(x) + lane_base;
    const float c2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    bool ok = true;
    // Waits ahead of warp-collective TMEM instructions: the whole warp proceeds or none of it.
    auto wait_warp = [&](uint64_t* bar, int phase) {
      const bool r = mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      return __all_sync(0xffffffffu, r);
    };
    // The two softmax warpgroups take turns on the exponentials (the MUFU-bound part), so
    // that one's TMEM traffic, row maxima and hand-offs -- and, with P aliasing S, its
    // P V and next S MMAs -- overlap the other's exponentials.  Round j is tile a's turn,
    // then tile b's; both run T = max(ta, tb) rounds per unit (a round without a tile only
    // passes the turn).  MUFU units belong to SM sub-partitions, and warp w of each warpgroup
    // runs on sub-partition w, so the turn passes between those two warps alone
    // (SDPA_SM_TURN_WARP) rather than between whole warpgroups.  my_turn completes once per
    // hand-over; tile b hands tile a its very first turn, and each unit's last hand-over from
    // b is tile a's first turn of the next unit.
    uint64_t* my_turn = &turn[SDPA_SM_TURN_WARP ? 4 * x + (warp & 3) : 4 * x];
    uint64_t* their_turn = &turn[SDPA_SM_TURN_WARP ? 4 * (x ^ 1) + (warp & 3) : 4 * (x ^ 1)];
    // SDPA_SM_TURN_NAMED: the turn passes through hardware named barriers instead (ids 1-8, one per
    // sub-partition and tile, 64 threads: the passing warp's bar.arrive and the taking warp's
    // bar.sync), whose release takes tens of clocks where an mbarrier wake-up took about 340.  A
    // named barrier cannot time out, so each warp runs exactly turn_total wait/pass pairs -- one
    // per round of every unit of this CTA, the same count for both warps of a pair -- even after a
    // failed wait: it then drops the work but keeps taking and passing its turns until the count is
    // reached, so its partner is never left at a barrier.  Tile b's very first pass is tile a's
    // first turn, and b's last pass, which no round would take, is not made.
    const int turn_mine = 1 + 4 * x + (warp & 3), turn_theirs = 1 + 4 * (x ^ 1) + (warp & 3);
    int R_turn = 0;  // the current round's turn phase (mbarrier turns)
    int turn_total = 0, turn_done = 0;
    if (SDPA_SM_TURN && SDPA_SM_TURN_NAMED)
      for (int k = 0, u = unit_of(0); u < n_units; u = unit_of(++k)) turn_total += unit_at(u).T;
    // (bar.sync / bar.arrive are whole-warp instructions: the warp is reconverged first, since the
    // per-row choice of exponential loop may have split it)
    auto turn_wait = [&]() -> bool {
      if (SDPA_SM_TURN_NAMED) {
        __syncwarp();
        named_bar_sync(turn_mine, 64);
        return true;
      }
      return wait_warp(my_turn, R_turn);
    };
    auto turn_pass = [&]() {
      if (SDPA_SM_TURN_NAMED) {
        __syncwarp();
        if (!(x == 1 && turn_done + 1 == turn_total)) named_bar_arrive(turn_theirs, 64);
        ++turn_done;
      } else {
        mbar_arrive(their_turn);
      }
    };
    if (SDPA_SM_TURN && x == 1) {
      if (!SDPA_SM_TURN_NAMED) mbar_arrive(their_turn);
      else if (turn_total > 0) {
        __syncwarp();
        named_bar_arrive(turn_theirs, 64);
      }
    }
    int rx = 0, R = 0, ox = 0;  // rounds of this tile so far, rounds of both, units with rounds
    for (int k = 0, u = unit_of(0); ok && u < n_units; u = unit_of(++k)) {
      const Unit g = unit_at(u);
      const int row = (x ? g.r0b : g.r0a) + t;
      const int tiles = x ? g.tb : g.ta;
      // keys this row may see: lo .. lim
      const int first = x ? g.fb : g.fa;
      int lim = p.n_kv - 1, lo = 0;
      {
        const long long pos = (long long)row + p.n_kv - p.n_q;
        if (win_right >= 0 && pos + win_right < lim) lim = (int)(pos + win_right < -1 ? -1 : pos + win_right);
        if (win_left >= 0 && pos - win_left > 0) lo = (int)(pos - win_left > p.n_kv ? p.n_kv : pos - win_left);
      }
      float m_u = NEG_INF;  // running max of scale*log2(e)*s
      float l = 0.f;
      for (int j = 0; ok && j < g.T; ++j) {
        R_turn = R + j;
        if (j >= tiles) {  // no key tile left for this query tile: only pass the turn
          if (SDPA_SM_TURN) {
            if (!(ok = turn_wait())) break;
            turn_pass();
          }
          continue;
        }
        uint32_t s[128];
        if (!(ok = wait_warp(&s_full[x], rx + j))) break;
        tc_fence_after_sync();
        tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
        tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
        tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&s[64]));
        tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&s[96]));
        tmem_wait_ld();
        reg_fence(s);
        if (C::SHARED_S) {  // S_x is in registers: the shared buffer may take the next S
          tc_fence_before_sync();
          __syncwarp();
          if (lane == 0) red_release_add(s_loads, 1u);
        } else if (C::P_SEPARATE) {  // S_x is in registers: the tensor core may overwrite it with the next S_x
          tc_fence_before_sync();
          mbar_arrive(&s_free[x]);
        }
        const int kv0 = (first + j) * 128;
        // Modes 0 and 1 have lo = 0, which kv0 + c >= 0 never falls below: one compare per score.
        const bool masked = kv0 + 127 > lim || (MASK == 2 && kv0 < lo);
        // With two exponential loops (d = 64) the loop is chosen per warp: a row of a masked tile
        // may itself see every key, and two loops in one warp would run one after the other.
        const bool warp_masked = C::POLY_EVERY > 0 ? __any_sync(0xffffffffu, masked) : masked;
        if (masked) {
          if (MASK == 2) {
            // Two-sided: per 32-column chunk, one mask of the hidden columns (below lo or above
            // lim), then a bit test and a select per score.
            const int hi = lim - kv0, lw = lo - kv0;  // this row sees columns lw .. hi
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int nb = min(max(lw - 32 * q, 0), 32);      // columns [0, nb) of the chunk are below lo
              const int na = min(max(hi - 32 * q + 1, 0), 32);  // columns [na, 32) are above lim
              const uint32_t below = nb >= 32 ? 0xffffffffu : (1u << nb) - 1u;
              const uint32_t kept = na >= 32 ? 0xffffffffu : (1u << na) - 1u;
              const uint32_t hidden = below | ~kept;
#pragma unroll
              for (int b = 0; b < 32; ++b)
                if (hidden & (1u << b)) s[32 * q + b] = __float_as_uint(NEG_INF);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (kv0 + c > lim) s[c] = __float_as_uint(NEG_INF);
          }
        }
        float mx;
        {  // eight independent chains of 3-input maxima over s[0..127]: 16 + 7 x 16 scores
          float m[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m[k] = fmaxf(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1]));
#pragma unroll
          for (int c = 16; c < 128; c += 16)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              m[k] = max3f(m[k], __uint_as_float(s[c + 2 * k]), __uint_as_float(s[c + 2 * k + 1]));
          mx = max3f(max3f(m[0], m[1], m[2]), max3f(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
        }
        const float m_new = fmaxf(m_u, mx * c2);
        const bool need = m_new > m_u + 8.0f;
        bool pv_waited = false;  // P_x V of the previous round known complete (P_x and O_x free)
        if (__any_sync(0xffffffffu, need)) {
          float alpha = 1.f;
          if (m_new > m_u) {
            alpha = ex2_approx(m_u - m_new);  // 0 when m_u = -inf
            m_u = m_new;
            l *= alpha;
          }
          if (j > 0) {  // O_x holds P V of earlier tiles of this unit
            if (C::P_SEPARATE) {
              if (!(ok = wait_warp(&pv_done[x], rx + j - 1))) break;
              tc_fence_after_sync();
              pv_waited = true;
            }  // (aliased P: S_x(j) was issued after P_x V of tile j-1, so that is complete)
#pragma unroll 1
            for (int cb = 0; cb < D; cb += 32) {
              uint32_t o[32];
              tmem_ld_32x32b_x32(tO + cb, o);
              tmem_wait_ld();
              reg_fence(o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st_32x32b_x32(tO + cb, o);
            }
          }
        }
        if (SDPA_SM_TURN && !(ok = turn_wait())) break;  // this warp's turn on the exponentials
        const float m_use = (m_u == NEG_INF) ? 0.f : m_u;
        uint32_t pk[64];
        l += warp_masked ? softmax_exp_row<0>(s, c2, m_use, pk) : softmax_exp_row<C::POLY_EVERY>(s, c2, m_use, pk);
        if (SDPA_SM_TURN) turn_pass();  // hand the exponentials over
        if (C::P_SEPARATE && rx + j > 0 && !pv_waited) {  // the last P_x V (this unit's or the previous one's) reads P_x
          if (!(ok = wait_warp(&pv_done[x], rx + j - 1))) break;
          tc_fence_after_sync();
        }
        tmem_st_32x32b_x32(tP + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st_32x32b_x32(tP + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_wait_st();
        tc_fence_before_sync();
#ifdef SDPA_FAULT_DROP_ARRIVE
        // Test builds only: tile b never reports its first P, so its MMA issuer's wait runs out.
        if (!(x == 1 && j == 0))
#endif
          mbar_arrive(&p_full[x]);
      }
      // ---------------------------------------------------------------- epilogue
      if (ok && tiles > 0) ok = wait_warp(&o_full[x], ox);
      if (ok) {
        tc_fence_after_sync();
        const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
        const bool store = row < p.n_q;
        uint4* orow = reinterpret_cast<uint4*>(p.O + ((size_t)g.bh * p.n_q + (store ? row : 0)) * D);
#pragma unroll 1
        for (int cb = 0; cb < D; cb += 32) {
          uint32_t o[32];
          if (tiles > 0) {
            tmem_ld_32x32b_x32(tO + cb, o);
            tmem_wait_ld();
            reg_fence(o);
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
          }
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
          if (store) {
#pragma unroll
            for (int v = 0; v < 4; ++v)
              orow[cb / 8 + v] = make_uint4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
          }
        }
        if (tiles > 0) {  // O_x has been read: the next unit's first P_x V may overwrite it
          tc_fence_before_sync();
          mbar_arrive(&o_free[x]);
        }
        if (store && p.LSE)
          p.LSE[(size_t)g.bh * p.n_q + row] = (l > 0.f) ? m_u * 0.69314718055994531f + logf(l) : NEG_INF;
      }
      rx += tiles;
      R += g.T;
      if (tiles > 0) ++ox;
    }
    // After a failed wait: the remaining turns, without the work (named barriers cannot time out)
    if (SDPA_SM_TURN && SDPA_SM_TURN_NAMED)
      while (turn_done < turn_total) {
        turn_wait();
        turn_pass();
      }
    if (SDPA_DEBUG && t == 0) dbg[2 + x] = rx, dbg[4 + x] = ox;
  }

  if (timed_out) record_error(6 /* SDPA_ERR_DEVICE_TIMEOUT */);
  tc_fence_before_sync();
  __syncthreads();
#if SDPA_DEBUG
  // Every barrier has completed exactly as many phases (mod 2) as its users counted: an arrive
  // too many or too few anywhere in the pipeline shows up here.
  if (threadIdx.x == 0 && !tmem_bad && !*abort_flag) {
    bool good = mbar_phase_is(q_full, dbg[0]) && mbar_phase_is(q_free, dbg[0]) && dbg[6] == dbg[0] &&
                dbg[7] == dbg[0];
    for (int s = 0; s < C::NSLOT; ++s) {
      const int n = dbg[1] > s ? (dbg[1] - s + C::NSLOT - 1) / C::NSLOT : 0;
      good = good && mbar_phase_is(&full[s], n) && mbar_phase_is(&empty[s], n);
    }
    for (int x = 0; x < 2; ++x) {
      const int rx = dbg[2 + x], ox = dbg[4 + x];
      good = good && mbar_phase_is(&s_full[x], rx) && mbar_phase_is(&p_full[x], rx) &&
             mbar_phase_is(&o_full[x], ox) && mbar_phase_is(&o_free[x], ox) && mbar_phase_is(&drain[x], 1);
      if (C::P_SEPARATE)
        good = good && mbar_phase_is(&s_free[x], C::SHARED_S ? 0 : rx) && mbar_phase_is(&pv_done[x], rx);
    }
    if (C::SHARED_S) good = good && *s_loads == 4u * (uint32_t)(dbg[2] + dbg[3]);
    if (!good) record_error(8 /* SDPA_ERR_DEVICE_CHECK */);
  }
#endif
  if (warp == C::MMA_WARP) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdpa
