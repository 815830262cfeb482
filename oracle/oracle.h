/*
 * Oracle for exact scaled dot-product attention: TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct CPU code in double precision.  Only the test
 * suite, the smoke check and the benchmark's CPU-baseline leg may load it; the
 * product library never does, and the two share no code.
 *
 * What it computes (the definition the attention pages derive from):
 *   Attention(Q, K, V) = softmax(Q K^T * scale) V, softmax taken row by row
 *   in its numerically stable, max-subtracted form
 *   ("Attention at the Theoretical Minimum: A Mathematics of Arrays Framework
 *   for Memory-Optimal Transformer Kernels", abstract; the agents-report.net
 *   MoA article, section "DNF derivation", where scale = 1/sqrt(d_k)).
 *
 * For one query row i of one (batch, head) slice:
 *   allowed(i, j) = true                          non-causal
 *                 = j <= i + (n_kv - n_q)         causal (bottom-right aligned)
 *                 = p - left <= j <= p + right    local window, p = i + (n_kv - n_q)
 *   s_ij  = scale * sum_k Q[i,k] K[j,k]           (allowed j only)
 *   m_i   = max_j s_ij
 *   e_ij  = exp(s_ij - m_i),  l_i = sum_j e_ij
 *   O[i,:] = (sum_j e_ij V[j,:]) / l_i
 *   LSE_i = m_i + ln l_i                          (natural log of the scaled logits)
 * A row with no allowed key gives O = 0 and LSE = -inf.
 *
 * Layout: row-major.  Q [n_q, d_k], K [n_kv, d_k], V [n_kv, d_v] per slice,
 * slices back to back ([bh, n, d]).  Inputs are float32: every bf16 and fp32
 * input value is exact in float32 and is widened exactly to double here.
 *
 * Grouped-query decode (several query heads reading one key/value head) is the
 * same definition with the key/value head chosen by the query head's group; the
 * 2-simplicial article (szyisi.cn, "model design") tiles along the query heads
 * of such groups to keep its kernels dense.
 *
 * The backward pass is the chain rule through the same definition: the
 * MoA roadmap's last stage is a DNF for the backward pass (agents-report.net MoA
 * article, "implementation roadmap"); its result is the ordinary gradient of exact
 * attention.
 *
 * Parity pins: see tests/test_oracle_pins.py (closed forms, invariants, brute
 * force, a hand-worked example and a library special case).
 */
#ifndef SDPA_ORACLE_H
#define SDPA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Full score matrix of one slice: S[i, j] = scale * q_i . k_j for allowed (i, j), -inf otherwise.
   S is [n_q, n_kv].  Returns 0 or -1 on a bad argument. */
int oracle_scores(const float* Q, const float* K, int64_t n_q, int64_t n_kv, int d_k, double scale,
                  int causal, double* S);

/* Row-wise softmax of an explicit matrix with the row maximum subtracted first.
   Entries equal to -inf get probability 0; a row that is all -inf becomes all zeros. */
int oracle_softmax_rows(const double* S, int64_t rows, int64_t cols, double* P);

/* The naive, unstable softmax exp(s) / sum exp(s) with NO max subtraction.
   Brute-force cross-check for small, well-scaled inputs only: it overflows for large logits. */
int oracle_softmax_naive(const double* S, int64_t rows, int64_t cols, double* P);

/* Full-matrix form for tiny problems: S (full), P = softmax_rows(S), O = P V, LSE.
   S_out and P_out may be NULL.  O is [n_q, d_v], LSE is [n_q]. */
int oracle_sdpa_full(const float* Q, const float* K, const float* V, int64_t n_q, int64_t n_kv, int d_k,
                     int d_v, double scale, int causal, double* S_out, double* P_out, double* O,
                     double* LSE);

/* Row-at-a-time form over bh independent slices, for the listed query rows of every slice.
   rows: n_rows indices in [0, n_q); NULL means all rows (n_rows must then equal n_q).
   O is [bh, n_rows, d_v], LSE is [bh, n_rows].  threads <= 0 means 1. */
int oracle_sdpa_rows(const float* Q, const float* K, const float* V, int64_t bh, int64_t n_q,
                     int64_t n_kv, int d_k, int d_v, double scale, int causal, const int64_t* rows,
                     int64_t n_rows, double* O, double* LSE, int threads);

/* oracle_sdpa_rows with a local window instead of the causal flag: query row i sits at key
   position p = i + (n_kv - n_q) and sees keys p - left <= j <= p + right; a negative bound
   leaves that side open ((-1, 0) is causal, (-1, -1) is full attention). */
int oracle_sdpa_rows_window(const float* Q, const float* K, const float* V, int64_t bh, int64_t n_q,
                            int64_t n_kv, int d_k, int d_v, double scale, int64_t left, int64_t right,
                            const int64_t* rows, int64_t n_rows, double* O, double* LSE, int threads);

/* Decode: one query row per (b, h) against the first lens[b] keys of a cache.
   Q [B, H, d_k]; K [B, H, n_cap, d_k]; V [B, H, n_cap, d_v]; O [B, H, d_v]; LSE [B, H].
   Only the (b, h) pairs listed in `pairs` (flat b*H + h, n_pairs of them) are computed, into
   O[p], LSE[p] in list order; pairs == NULL means all B*H pairs in order. */
int oracle_decode(const float* Q, const float* K, const float* V, const int32_t* lens, int64_t B,
                  int64_t H, int64_t n_cap, int d_k, int d_v, double scale, const int64_t* pairs,
                  int64_t n_pairs, double* O, double* LSE, int threads);

/* Grouped-query decode: H_q query heads share H_kv key/value heads (H_q a multiple of H_kv),
   query head h reading key/value head h / (H_q / H_kv) -- consecutive query heads form a group.
   Q [B, H_q, d_k]; K [B, H_kv, n_cap, d_k]; V [B, H_kv, n_cap, d_v]; O [B, H_q, d_v]; LSE [B, H_q].
   pairs: flat b*H_q + h indices as in oracle_decode (NULL = all, in order).  H_kv == H_q is
   oracle_decode. */
int oracle_decode_gqa(const float* Q, const float* K, const float* V, const int32_t* lens, int64_t B,
                      int64_t H_q, int64_t H_kv, int64_t n_cap, int d_k, int d_v, double scale,
                      const int64_t* pairs, int64_t n_pairs, double* O, double* LSE, int threads);

/* Backward pass of one (batch, head) slice at a time, for the forward above (causal or not).
   With P = softmax_rows(S) and loss gradient dO = dL/dO:
     dV = P^T dO;  dP = dO V^T;  dS_ij = P_ij (dP_ij - sum_k P_ik dP_ik);
     dQ = scale dS K;  dK = scale dS^T Q.
   Every query row is visited (each row's softmax is needed for every key column); only the
   listed outputs are written: dQ rows q_rows (n_qr of them, NULL = all n_q in order) into
   dQ [bh, n_qr, d_k]; dK and dV rows k_rows (NULL = all n_kv) into dK [bh, n_kr, d_k] and
   dV [bh, n_kr, d_v].  Output pointers may be NULL to skip that output.  A row with no
   allowed key contributes nothing.  threads <= 0 means 1. */
int oracle_sdpa_backward(const float* Q, const float* K, const float* V, const float* dO, int64_t bh,
                         int64_t n_q, int64_t n_kv, int d_k, int d_v, double scale, int causal,
                         const int64_t* q_rows, int64_t n_qr, const int64_t* k_rows, int64_t n_kr, double* dQ,
                         double* dK, double* dV, int threads);

#ifdef __cplusplus
}
#endif

#endif
