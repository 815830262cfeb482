// decode_gqa.cuh -- grouped-query decode on the sm_100a tensor cores.
//
// With grouped-query attention, G = H_q / H_kv consecutive query heads read one
// key/value head.  Tiling along the query heads of a group turns decode's
// matrix-vector products into small dense matrix products (the 2-simplicial
// article, szyisi.cn, "model design", uses a large grouped-query ratio for
// exactly that): each key and value row is read from HBM once and used by all
// G heads, so the kernel stays a bandwidth-bound stream while the tensor core
// does the G-fold arithmetic.
//
// CTA (split s, key/value head kvh, batch b) reduces keys [s*chunk, s*chunk+chunk)
// of the valid prefix [0, len_b) to a partial (O_s normalised, lse_s) per query
// head of the group; sdpa_decode_combine_kernel merges the splits.  Per 128-key
// tile j, with the group's queries padded to NQ rows (NQ = 16 or 32):
//   S^T = K_j Q^T         tcgen05.mma M = 128 keys, N = NQ heads, K = 128 dims
//   p   = 2^(S^T * scale * log2 e - m)   one thread per key (TMEM lane = key)
//   O^T += V_j^T P^T      tcgen05.mma M = 128 dims, N = NQ heads, K = 128 keys
// S^T and O^T live in TMEM; P^T goes to shared memory (a tcgen05 B operand).
// The reference maximum m of each head is shared by the CTA's 128 key threads
// and changes only when a score exceeds it by more than 8 (a factor 256): a
// vote (barrier.red.or) detects that, and only then is the per-head maximum
// reduced and O^T rescaled.  O^T and the per-thread sums always share the same
// reference, so the result is exact whatever reference is used.
//
// Warp roles (192 threads): warp 0 TMA producer (Q once, then K_j, V_j into a
// ring of NSLOT 32 KB slots -- six, so three K/V tile pairs are in flight from
// HBM), warp 1 MMA issuer and TMEM owner, warps 2-5 the softmax (one key each)
// and the epilogue (one output dimension each).
#pragma once

#include <cuda_bf16.h>

#include "sm100.cuh"
#include "decode.cuh"

#ifndef SDPA_GQA_CHUNK_MAX
#define SDPA_GQA_CHUNK_MAX 4096  // measured on 64 x (64 over 8 heads), 16384 cache: 2048 5.94, 4096 6.22, 8192 6.15 TB/s
#endif
#ifndef SDPA_GQA_NSLOT
#define SDPA_GQA_NSLOT 6  // 192 KB of ring, one CTA per SM (measured: 6 slots 5.94, 3 slots x 2 CTAs 5.70 TB/s)
#endif

namespace sdpa {

template <int NQ>  // query heads per MMA (the group, padded)
struct GqaCfg {
  static_assert(NQ == 16 || NQ == 32, "NQ is 16 or 32");
  static constexpr int D = 128;
  static constexpr int TILE_BYTES = 128 * D * 2;     // 128 keys x 128 dims, bf16
  static constexpr int BLOCK_BYTES = 128 * 64 * 2;   // one 64-dim swizzle block of a tile
  static constexpr int NSLOT = SDPA_GQA_NSLOT;       // ring slots: K_0, V_0, K_1, V_1, ...
  static constexpr int QP_BLOCK = NQ * 128;          // NQ rows x 64 bf16 (a block of Q or of P^T)
  static constexpr int KV_OFF = 0;
  static constexpr int Q_OFF = NSLOT * TILE_BYTES;
  static constexpr int P_OFF = Q_OFF + 2 * QP_BLOCK;  // two P^T buffers of two blocks
  static constexpr int BAR_OFF = P_OFF + 4 * QP_BLOCK;
  // q_full, full[NSLOT], empty[NSLOT], s_full[2], s_free[2], p_full[2], pv_done[2], drain
  static constexpr int NBAR = 1 + 2 * NSLOT + 8 + 1;
  static constexpr int RED_OFF = BAR_OFF + NBAR * 8 + 16;  // after the TMEM slot and abort flag
  static constexpr int SMEM_BYTES = RED_OFF + 4 * NQ * 4 + 1024;
  static constexpr int THREADS = 192;
  static constexpr int MIN_BLOCKS = (NQ == 16 && NSLOT <= 3) ? 2 : 1;  // two CTAs per SM fit 3 slots each
  static constexpr uint32_t TMEM_COLS = (3 * NQ <= 64) ? 64u : 128u;
  static constexpr uint32_t COL_O = 2 * NQ;  // S^T buffers at columns [0, NQ) and [NQ, 2 NQ)
};

// Keys per split (a multiple of 128): the largest of SDPA_GQA_CHUNK_MAX .. 128 whose grid over the
// full cache still has 4 CTAs per SM.  Longer splits mean fewer CTA start-ups (barrier set-up,
// TMEM allocation, the first loads' latency) per byte streamed.
__host__ __device__ inline int gqa_chunk(long long batch, long long heads_kv, long long n_cap) {
  int chunk = SDPA_GQA_CHUNK_MAX;
  while (chunk > 128 && batch * heads_kv * ((n_cap + chunk - 1) / chunk) < 148LL * 4) chunk >>= 1;
  return chunk;
}

struct GqaParams {
  float* part_o;       // [B, H_q, n_split, 128]
  float* part_lse;     // [B, H_q, n_split], natural log
  const int* kv_lens;  // [B]
  int H_q, H_kv, group, n_cap, chunk, n_split;
  float scale_log2;    // scale * log2(e)
};

template <int NQ>
__global__ void __launch_bounds__(192, GqaCfg<NQ>::MIN_BLOCKS)
    sdpa_decode_gqa_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const GqaParams p) {
  using C = GqaCfg<NQ>;
  using namespace sm100;
  const int s = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int len = decode_len(p.kv_lens, b, p.n_cap);
  const int k_begin = s * p.chunk;
  if (k_begin >= len) return;  // the whole CTA: nothing of this split is valid
  const int k_end = min(k_begin + p.chunk, len);
  const int T = (k_end - k_begin + 127) / 128;
  const int G = p.group;
  const int bkv = b * p.H_kv + kvh;        // key/value slice
  const int q_row0 = b * p.H_q + kvh * G;  // the group's first query head, a row of [B*H_q, 128]

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sKV = smem + C::KV_OFF;
  uint8_t* sQ = smem + C::Q_OFF;
  uint8_t* sP = smem + C::P_OFF;
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* full = bars + 1;
  uint64_t* empty = full + C::NSLOT;
  uint64_t* s_full = empty + C::NSLOT;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 2;
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = (uint32_t*)(bars + C::NBAR);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  float* red = (float*)(smem + C::RED_OFF);  // [4 warps][NQ]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&s_free[x], 128);
      mbar_init(&p_full[x], 128);
      mbar_init(&pv_done[x], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  bool timed_out = false;
  const bool tmem_bad = tmem_alloc_bad(tmem);  // debug builds only

  if (tmem_bad) {
  } else if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * C::QP_BLOCK);
      tma_load_3d(sQ, &tmQ, q_full, 0, q_row0, 0);
      tma_load_3d(sQ + C::QP_BLOCK, &tmQ, q_full, 64, q_row0, 0);
      int issued = 0;
      for (int idx = 0; idx < 2 * T; ++idx) {
        const int slot = idx % C::NSLOT;
        const uint32_t ph = (uint32_t)(idx / C::NSLOT) & 1u;
        if (!mbar_wait_bounded(&empty[slot], ph ^ 1u, abort_flag, &timed_out)) break;
        mbar_arrive_expect_tx(&full[slot], C::TILE_BYTES);
        const CUtensorMap* map = (idx & 1) ? &tmV : &tmK;
        uint8_t* dst = sKV + slot * C::TILE_BYTES;
        const int key0 = k_begin + (idx >> 1) * 128;
        tma_load_3d(dst, map, &full[slot], 0, key0, bkv);
        tma_load_3d(dst + C::BLOCK_BYTES, map, &full[slot], 64, key0, bkv);
        issued = idx + 1;
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        mbar_wait_drain(q_full, 0);
        for (int idx = (issued > C::NSLOT ? issued - C::NSLOT : 0); idx < issued; ++idx)
          mbar_wait_drain(&full[idx % C::NSLOT], (uint32_t)(idx / C::NSLOT) & 1u);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, NQ, false, false);  // K (K-major) x Q (K-major)
      constexpr uint32_t idO = idesc_bf16_f32(128, NQ, true, false);   // V^T (MN-major) x P^T (K-major)
      const uint32_t sKVa = smem_u32(sKV);
      const uint64_t dK = smem_desc_sw128(sKVa, 16, 1024);
      const uint64_t dV = smem_desc_sw128(sKVa, C::BLOCK_BYTES, 1024);
      const uint64_t dQ = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dP = smem_desc_sw128(smem_u32(sP), 16, 1024);
      auto issue_S = [&](int t) {  // S^T(t) = K_t Q^T into S buffer t & 1
        const uint64_t a0 = dK + (uint64_t)((((2 * t) % C::NSLOT) * C::TILE_BYTES) >> 4);
        const uint32_t d = tmem + (uint32_t)((t & 1) * NQ);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t oa = (uint64_t)((((kk >> 2) * C::BLOCK_BYTES) + (kk & 3) * 32) >> 4);
          const uint64_t ob = (uint64_t)((((kk >> 2) * C::QP_BLOCK) + (kk & 3) * 32) >> 4);
          mma_ss(d, a0 + oa, dQ + ob, idS, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_PV = [&](int t) {  // O^T += V_t^T P^T(t)
        const uint64_t a0 = dV + (uint64_t)((((2 * t + 1) % C::NSLOT) * C::TILE_BYTES) >> 4);
        const uint64_t b0 = dP + (uint64_t)(((t & 1) * 2 * C::QP_BLOCK) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t ob = (uint64_t)((((kk >> 2) * C::QP_BLOCK) + (kk & 3) * 32) >> 4);
          mma_ss(tmem + C::COL_O, a0 + (uint64_t)((kk * 2048) >> 4), b0 + ob, idO, (t > 0 || kk > 0) ? 1u : 0u);
        }
      };
      auto wait_bar = [&](uint64_t* bar, int phase) {
        return mbar_wait_bounded(bar, (uint32_t)phase & 1u, abort_flag, &timed_out);
      };
      auto wait_slot = [&](int idx) { return wait_bar(&full[idx % C::NSLOT], idx / C::NSLOT); };

      bool ok = wait_bar(q_full, 0) && wait_slot(0);
      if (ok) {
        issue_S(0);
        tc_commit(&s_full[0]);
        tc_commit(&empty[0]);
      }
      for (int t = 0; ok && t < T; ++t) {
        if (t + 1 < T) {  // keep the next scores ahead of this tile's P V
          const int u = t + 1;
          if (!(ok = wait_slot(2 * u) && (u < 2 || wait_bar(&s_free[u & 1], (u - 2) >> 1)))) break;
          issue_S(u);
          tc_commit(&s_full[u & 1]);
          tc_commit(&empty[(2 * u) % C::NSLOT]);
        }
        if (!(ok = wait_slot(2 * t + 1) && wait_bar(&p_full[t & 1], t >> 1))) break;
        issue_PV(t);
        tc_commit(&pv_done[t & 1]);
        tc_commit(&empty[(2 * t + 1) % C::NSLOT]);
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax and epilogue
    const int q4 = warp & 3;          // TMEM lane quarter this warp may access
    const int row = 32 * q4 + lane;   // TMEM lane: the tile's key (softmax), the dimension (epilogue)
    const int tid = threadIdx.x - 64;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
    const float c2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    float m_ref[NQ], l_part[NQ];
#pragma unroll
    for (int g = 0; g < NQ; ++g) {
      m_ref[g] = NEG_INF;
      l_part[g] = 0.f;
    }
    // P^T columns of padded heads (g >= G) are never written again: zero both buffers once.
    for (int i = tid; i < C::QP_BLOCK / 4; i += 128) reinterpret_cast<uint4*>(sP)[i] = make_uint4(0, 0, 0, 0);

    bool ok = true;
    for (int t = 0; t < T; ++t) {
      const int buf = t & 1;
      const bool w = __all_sync(0xffffffffu, mbar_wait_bounded(&s_full[buf], (uint32_t)(t >> 1) & 1u, abort_flag,
                                                                 &timed_out));
      if (named_bar_any(1, 128, !(w && ok))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t sr[NQ];
#pragma unroll
      for (int c = 0; c < NQ / 16; ++c)
        tmem_ld_32x32b_x16(tmem + (uint32_t)(buf * NQ + 16 * c) + lane_base,
                           *reinterpret_cast<uint32_t(*)[16]>(&sr[16 * c]));
      tmem_wait_ld();
      reg_fence(sr);
      tc_fence_before_sync();
      mbar_arrive(&s_free[buf]);

      const bool valid = k_begin + t * 128 + row < k_end;
      float v[NQ];
      bool need = false;
#pragma unroll
      for (int g = 0; g < NQ; ++g) {
        v[g] = (valid && g < G) ? __uint_as_float(sr[g]) * c2 : NEG_INF;
        need |= v[g] > m_ref[g] + 8.f;
      }
      if (named_bar_any(1, 128, need)) {  // a score outgrew its head's reference: move it
        float alpha[NQ];
#pragma unroll
        for (int g = 0; g < NQ; ++g) {
          float x = v[g];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
          if (lane == 0) red[q4 * NQ + g] = x;
        }
        named_bar_sync(2, 128);
#pragma unroll
        for (int g = 0; g < NQ; ++g) {
          const float tm = fmaxf(fmaxf(red[g], red[NQ + g]), fmaxf(red[2 * NQ + g], red[3 * NQ + g]));
          const float mn = fmaxf(m_ref[g], tm);
          alpha[g] = (m_ref[g] == NEG_INF) ? 0.f : ex2_approx(m_ref[g] - mn);
          m_ref[g] = mn;
          l_part[g] *= alpha[g];
        }
        named_bar_sync(2, 128);  // every thread has read `red`
        if (t > 0) {  // O^T holds P V of tiles 0 .. t-1: rescale it once they are complete
          const bool w2 = __all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[(t - 1) & 1],
                                                                    (uint32_t)((t - 1) >> 1) & 1u, abort_flag,
                                                                    &timed_out));
          if (w2) {
            tc_fence_after_sync();
#pragma unroll
            for (int c = 0; c < NQ / 16; ++c) {
              uint32_t o[16];
              const uint32_t ta = tmem + C::COL_O + (uint32_t)(16 * c) + lane_base;
              tmem_ld_32x32b_x16(ta, o);
              tmem_wait_ld();
              reg_fence(o);
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[16 * c + i]);
              tmem_st_32x32b_x16(ta, o);
            }
            tmem_wait_st();
          } else {
            ok = false;
          }
        }
      }
      // P^T buffer `buf` was last read by P V of tile t - 2
      if (t >= 2 && !__all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[buf], (uint32_t)((t - 2) >> 1) & 1u,
                                                                abort_flag, &timed_out)))
        ok = false;
      uint8_t* pb = sP + buf * 2 * C::QP_BLOCK + (row >> 6) * C::QP_BLOCK;
      const int cb = (row & 63) * 2;  // byte column of this key in its 128-byte row
#pragma unroll
      for (int g = 0; g < NQ; ++g) {
        if (g < G) {
          const float m_use = (m_ref[g] == NEG_INF) ? 0.f : m_ref[g];
          const float e = ex2_approx(v[g] - m_use);
          l_part[g] += e;
          // 128-byte swizzle: 16-byte chunk index XOR (row & 7), rows 128 bytes apart
          *reinterpret_cast<__nv_bfloat16*>(pb + g * 128 + ((((cb >> 4) ^ (g & 7)) << 4) | (cb & 15))) =
              __float2bfloat16_rn(e);
        }
      }
      if (!valid) {
        // Past the split's last key the cache rows may hold anything (NaN): P is 0 there, but
        // 0 * NaN is NaN, so this key's V row is zeroed once it has landed.
        const int idx = 2 * t + 1;
        if (mbar_wait_bounded(&full[idx % C::NSLOT], (uint32_t)(idx / C::NSLOT) & 1u, abort_flag, &timed_out)) {
          uint4* r0 = reinterpret_cast<uint4*>(sKV + (idx % C::NSLOT) * C::TILE_BYTES + row * 128);
          uint4* r1 = reinterpret_cast<uint4*>(sKV + (idx % C::NSLOT) * C::TILE_BYTES + C::BLOCK_BYTES + row * 128);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            r0[i] = make_uint4(0, 0, 0, 0);
            r1[i] = make_uint4(0, 0, 0, 0);
          }
        } else {
          ok = false;
        }
      }
      fence_proxy_async_smem();  // P^T and zeroed rows: visible to the tensor core
      tc_fence_before_sync();
      mbar_arrive(&p_full[buf]);
    }

    // ------------------------------------------------------------------ epilogue
    if (ok)
      ok = __all_sync(0xffffffffu, mbar_wait_bounded(&pv_done[(T - 1) & 1], (uint32_t)((T - 1) >> 1) & 1u,
                                                     abort_flag, &timed_out));
    if (!named_bar_any(1, 128, !ok)) {
      tc_fence_after_sync();
#pragma unroll
      for (int g = 0; g < NQ; ++g) {  // per-head sums over the 128 key threads
        float x = l_part[g];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        if (lane == 0) red[q4 * NQ + g] = x;
      }
      named_bar_sync(2, 128);
      uint32_t o[NQ];
#pragma unroll
      for (int c = 0; c < NQ / 16; ++c)
        tmem_ld_32x32b_x16(tmem + C::COL_O + (uint32_t)(16 * c) + lane_base,
                           *reinterpret_cast<uint32_t(*)[16]>(&o[16 * c]));
      tmem_wait_ld();
      reg_fence(o);
#pragma unroll
      for (int g = 0; g < NQ; ++g) {
        if (g < G) {
          const float l = red[g] + red[NQ + g] + red[2 * NQ + g] + red[3 * NQ + g];
          const size_t part = ((size_t)(b * p.H_q + kvh * G + g)) * p.n_split + s;
          p.part_o[part * 128 + row] = __uint_as_float(o[g]) / l;  // row = output dimension here
          if (row == g) p.part_lse[part] = (m_ref[g] + log2f(l)) * 0.69314718055994531f;
        }
      }
    }
  }

  if (timed_out) record_error(6 /* SDPA_ERR_DEVICE_TIMEOUT */);
  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace sdpa
