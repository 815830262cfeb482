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
//   warp  9    MMA issuer (one thread) and TMEM owner
//   warps 10-11 idle
// Registers: each SM sub-partition holds 16K 32-bit registers and receives
// one warp of every warpgroup, so the CTA launches at 168 per thread and then
// moves registers from the producer/MMA warpgroup (down to 56) to the two
// softmax warpgroups (up to 224): 2*224 + 56 <= 512 per sub-partition lane
// slot, and 56*128 + 224*256 = 384*168 in total.
// TMEM (512 columns): S_a [0,128), S_b [128,256), O_a [256,256+D), O_b [384,384+D).
// P_x (bf16, two per column) overwrites the first 64 columns of S_x once the
// softmax has read S_x; the next S_x MMA is issued after the P_x V MMA, and
// tcgen05 MMAs from one thread run in issue order.
//
// Per key tile j the issuer runs PV_a(j), S_a(j+1), PV_b(j), S_b(j+1), so that
// one softmax warpgroup works while the tensor core serves the other.  The
// online softmax keeps, per row, the running maximum m (in log2 units of the
// scaled logits) and sum l; O and l are rescaled only when m grows by more
// than 8 (a factor 256): O and l always share the same reference maximum, so
// O/l is exact whatever reference is used, and fp32 cannot overflow.
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sdpa {

template <int D>
struct PrefillCfg {
  static constexpr int BM = 128;                        // query rows per tile
  static constexpr int BN = 128;                        // key rows per tile
  static constexpr int TILE_BYTES = 128 * D * 2;        // one 128 x D bf16 tile
  static constexpr int BLOCK_BYTES = 128 * 64 * 2;      // one 128-row x 64-column swizzle block (16 KB)
  static constexpr int NSLOT = (D == 128) ? 4 : 8;      // K/V ring slots
  static constexpr int Q_OFF = 0;
  static constexpr int KV_OFF = 2 * TILE_BYTES;
  static constexpr int BAR_OFF = KV_OFF + NSLOT * TILE_BYTES;
  static constexpr int NBAR = 1 + 2 * NSLOT + 2 + 2 + 2 + 1;
  static constexpr int SMEM_BYTES = BAR_OFF + NBAR * 8 + 16 + 1024;  // + tmem slot, abort flag, align slack
  static constexpr int THREADS = 384;
  static constexpr int SOFTMAX_REGS = 224;
  static constexpr int CONTROL_REGS = 56;
  static constexpr int LOAD_WARP = 8;
  static constexpr int MMA_WARP = 9;
  static constexpr uint32_t TMEM_COLS = 512;
};

__device__ int g_sdpa_error;  // first device-side error since the last read (0 = none)

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_sdpa_error, 0, code); }

// Number of 128-row key tiles query tile [r0, r0+128) must visit.
__host__ __device__ inline int prefill_kv_tiles(int r0, int n_q, int n_kv, bool causal) {
  if (r0 >= n_q) return 0;
  const int total = (n_kv + 127) / 128;
  if (!causal) return total;
  const int last_row = (r0 + 127 < n_q - 1) ? r0 + 127 : n_q - 1;
  const long long max_key = (long long)last_row + n_kv - n_q;  // bottom-right aligned
  if (max_key < 0) return 0;
  const int t = (int)(max_key / 128) + 1;
  return t < total ? t : total;
}

struct PrefillParams {
  __nv_bfloat16* O;
  float* LSE;
  int n_q, n_kv, bh_count, n_pairs;
  float scale_log2;  // scale * log2(e), > 0
};

template <int D, bool CAUSAL>
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
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: heaviest query-tile pairs (the last rows, under a causal mask) first.
  const int bh = blockIdx.x % p.bh_count;
  const int pair = p.n_pairs - 1 - (int)(blockIdx.x / p.bh_count);
  const int r0a = pair * 256, r0b = pair * 256 + 128;
  const int ta = prefill_kv_tiles(r0a, p.n_q, p.n_kv, CAUSAL);
  const int tb = prefill_kv_tiles(r0b, p.n_q, p.n_kv, CAUSAL);
  const int T = ta > tb ? ta : tb;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::NSLOT; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_full[x], 1);
    }
    mbar_init(drain, 1);
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
  static_assert(C::SOFTMAX_REGS * 256 + C::CONTROL_REGS * 128 <= 168 * 384, "register split exceeds the launch");
  if (warp >= 8) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::CONTROL_REGS));
    if (warp == C::LOAD_WARP) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && T > 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        mbar_arrive_expect_tx(q_full, 2 * C::TILE_BYTES);
  #pragma unroll
        for (int x = 0; x < 2; ++x)
  #pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(sQ + x * C::TILE_BYTES + cb * C::BLOCK_BYTES, &tmQ, q_full, cb * 64, x ? r0b : r0a, bh);
        int issued = 0;
        for (int idx = 0; idx < 2 * T; ++idx) {
          const int slot = idx % C::NSLOT;
          const uint32_t ph = (uint32_t)(idx / C::NSLOT) & 1u;
          if (!mbar_wait_bounded(&empty[slot], ph ^ 1u, abort_flag, &timed_out)) break;
          mbar_arrive_expect_tx(&full[slot], C::TILE_BYTES);
          const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
          uint8_t* dst = sKV + slot * C::TILE_BYTES;
  #pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_3d(dst + cb * C::BLOCK_BYTES, map, &full[slot], cb * 64, (idx >> 1) * 128, bh);
          issued = idx + 1;
        }
        if (*abort_flag) {  // let the copies already in flight land before the CTA exits
          mbar_wait_drain(q_full, 0);
          for (int idx = (issued > C::NSLOT ? issued - C::NSLOT : 0); idx < issued; ++idx)
            mbar_wait_drain(&full[idx % C::NSLOT], (uint32_t)(idx / C::NSLOT) & 1u);
        }
      }
    } else if (warp == C::MMA_WARP) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0 && T > 0) {
        const uint32_t tS[2] = {tmem + 0u, tmem + 128u};
        const uint32_t tO[2] = {tmem + 256u, tmem + 384u};
        constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
        constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);     // P (TMEM) x V (MN-major)
        const uint32_t sQa = smem_u32(sQ), sKVa = smem_u32(sKV);

        auto issue_S = [&](int x, int j) {  // S_x = Q_x K_j^T
          const uint32_t qa = sQa + x * C::TILE_BYTES;
          const uint32_t ka = sKVa + ((2 * j) % C::NSLOT) * C::TILE_BYTES;
  #pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * C::BLOCK_BYTES + (kk & 3) * 32;
            mma_ss(tS[x], smem_desc_sw128(qa + off, 16, 1024), smem_desc_sw128(ka + off, 16, 1024), idS,
                   kk > 0 ? 1u : 0u);
          }
        };
        auto issue_PV = [&](int x, int j) {  // O_x += P_x V_j
          const uint32_t va = sKVa + ((2 * j + 1) % C::NSLOT) * C::TILE_BYTES;
  #pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            mma_ts(tO[x], tS[x] + kk * 8, smem_desc_sw128(va + kk * 2048, C::BLOCK_BYTES, 1024), idO,
                   (j > 0 || kk > 0) ? 1u : 0u);
        };
        auto wait_slot = [&](int idx) {
          return mbar_wait_bounded(&full[idx % C::NSLOT], (uint32_t)(idx / C::NSLOT) & 1u, abort_flag,
                                   &timed_out);
        };

        bool ok = mbar_wait_bounded(q_full, 0, abort_flag, &timed_out) && wait_slot(0);
        if (ok) {
          tc_fence_after_sync();
          if (ta > 0) { issue_S(0, 0); tc_commit(&s_full[0]); }
          if (tb > 0) { issue_S(1, 0); tc_commit(&s_full[1]); }
          tc_commit(&empty[0]);
        }
        for (int j = 0; ok && j < T; ++j) {
          if (!(ok = wait_slot(2 * j + 1))) break;  // V_j
          tc_fence_after_sync();
          if (j < ta) {
            if (!(ok = mbar_wait_bounded(&p_full[0], (uint32_t)j & 1u, abort_flag, &timed_out))) break;
            tc_fence_after_sync();
            issue_PV(0, j);
            if (j == ta - 1) tc_commit(&o_full[0]);
          }
          if (j + 1 < T) {
            if (!(ok = wait_slot(2 * (j + 1)))) break;  // K_{j+1}
            tc_fence_after_sync();
            if (j + 1 < ta) { issue_S(0, j + 1); tc_commit(&s_full[0]); }
          }
          if (j < tb) {
            if (!(ok = mbar_wait_bounded(&p_full[1], (uint32_t)j & 1u, abort_flag, &timed_out))) break;
            tc_fence_after_sync();
            issue_PV(1, j);
            if (j == tb - 1) tc_commit(&o_full[1]);
          }
          tc_commit(&empty[(2 * j + 1) % C::NSLOT]);  // V_j slot free once both PV MMAs are done
          if (j + 1 < T) {
            if (j + 1 < tb) { issue_S(1, j + 1); tc_commit(&s_full[1]); }
            tc_commit(&empty[(2 * (j + 1)) % C::NSLOT]);  // K_{j+1} slot
          }
        }
        // Every MMA and every commit issued above has landed before TMEM is released
        // and before the CTA's shared memory (which the commits arrive on) goes away.
        tc_commit(drain);
        mbar_wait_drain(drain, 0);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::SOFTMAX_REGS));
    // ------------------------------------------------ softmax + epilogue warpgroups
    const int x = warp >> 2;  // query tile a (0) or b (1)
    const int t = threadIdx.x & 127;
    const int row = (x ? r0b : r0a) + t;
    const int tiles = x ? tb : ta;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + (x ? 128u : 0u) + lane_base;
    const uint32_t tO = tmem + (x ? 384u : 256u) + lane_base;
    // last key this row may see
    int lim = p.n_kv - 1;
    if (CAUSAL) {
      const long long c = (long long)row + p.n_kv - p.n_q;
      if (c < lim) lim = (int)(c < -1 ? -1 : c);
    }
    const float c2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m_u = NEG_INF;  // running max of scale*log2(e)*s
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < tiles; ++j) {
      if (!(ok = mbar_wait_bounded(&s_full[x], (uint32_t)j & 1u, abort_flag, &timed_out))) break;
      tc_fence_after_sync();
      uint32_t s[128];
      {
        uint32_t(&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
        uint32_t(&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
        uint32_t(&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
        uint32_t(&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
        tmem_ld_32x32b_x32(tS + 0, s0);
        tmem_ld_32x32b_x32(tS + 32, s1);
        tmem_ld_32x32b_x32(tS + 64, s2);
        tmem_ld_32x32b_x32(tS + 96, s3);
        tmem_wait_ld();
        reg_fence(s);
      }
      const int kv0 = j * 128;
      if (kv0 + 127 > lim) {
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (kv0 + c > lim) s[c] = __float_as_uint(NEG_INF);
      }
      float mx = NEG_INF;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(s[c]));
      const float m_new = fmaxf(m_u, mx * c2);
      const bool need = m_new > m_u + 8.0f;
      if (__any_sync(0xffffffffu, need)) {
        float alpha = 1.f;
        if (m_new > m_u) {
          alpha = ex2_approx(m_u - m_new);  // 0 when m_u = -inf
          m_u = m_new;
          l *= alpha;
        }
        if (j > 0) {  // O_x holds PV of earlier tiles (complete: S_x(j) was issued after them)
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
      const float m_use = (m_u == NEG_INF) ? 0.f : m_u;
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 128; c += 2) {
        const float p0 = ex2_approx(fmaf(__uint_as_float(s[c]), c2, -m_use));
        const float p1 = ex2_approx(fmaf(__uint_as_float(s[c + 1]), c2, -m_use));
        rs += p0 + p1;
        pk[c >> 1] = pack_bf16x2(p0, p1);
      }
      l += rs;
      tmem_st_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      tmem_st_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&p_full[x]);
    }
    // ---------------------------------------------------------------- epilogue
    if (ok && tiles > 0) ok = mbar_wait_bounded(&o_full[x], 0, abort_flag, &timed_out);
    if (ok) {
      tc_fence_after_sync();
      const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
      const bool store = row < p.n_q;
      uint4* orow = reinterpret_cast<uint4*>(p.O + ((size_t)bh * p.n_q + (store ? row : 0)) * D);
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
      if (store && p.LSE)
        p.LSE[(size_t)bh * p.n_q + row] = (l > 0.f) ? m_u * 0.69314718055994531f + logf(l) : NEG_INF;
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

}  // namespace sdpa
