// Oracle for exact scaled dot-product attention -- TEST INFRASTRUCTURE ONLY.
// See oracle.h for the definition it follows and its citations.  Plain C++17,
// double precision, one score row at a time (the shape of the MoA article's
// C example: per query row, an O(n) vector of scores, its maximum, the
// exponentials, their sum, then the output row), or the full matrix for tiny
// problems.  No blocking, fusion or reordering beyond the definition.
#include "oracle.h"

#include <cmath>
#include <limits>
#include <thread>
#include <vector>

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

bool allowed(int64_t i, int64_t j, int64_t n_q, int64_t n_kv, int causal) {
  if (!causal) return true;
  return j <= i + (n_kv - n_q);  // bottom-right aligned causal mask
}

// Local window: query row i sits at key position p = i + (n_kv - n_q) and sees keys
// p - left <= j <= p + right; a negative bound means that side is unbounded.
bool allowed_window(int64_t i, int64_t j, int64_t n_q, int64_t n_kv, int64_t left, int64_t right) {
  const int64_t pos = i + (n_kv - n_q);
  if (left >= 0 && j < pos - left) return false;
  if (right >= 0 && j > pos + right) return false;
  return true;
}

// s_j = scale * q . k_j for every key j of one slice; -inf where masked.
// causal < 0 selects the local window (left, right) instead of the causal flag.
void score_row(const float* Q, const float* K, int64_t i, int64_t n_q, int64_t n_kv, int d_k,
               double scale, int causal, double* s, int64_t left = -1, int64_t right = -1) {
  const float* q = Q + i * d_k;
  for (int64_t j = 0; j < n_kv; ++j) {
    const bool ok = causal >= 0 ? allowed(i, j, n_q, n_kv, causal) : allowed_window(i, j, n_q, n_kv, left, right);
    if (!ok) {
      s[j] = kNegInf;
      continue;
    }
    const float* k = K + j * d_k;
    double dot = 0.0;
    for (int c = 0; c < d_k; ++c) dot += (double)q[c] * (double)k[c];
    s[j] = scale * dot;
  }
}

// Stable softmax of one row: p_j = exp(s_j - m) / sum_j exp(s_j - m).
// Returns m and l = sum_j exp(s_j - m) through the pointers (m = -inf, l = 0 if all masked).
void softmax_row(const double* s, int64_t n, double* p, double* m_out, double* l_out) {
  double m = kNegInf;
  for (int64_t j = 0; j < n; ++j)
    if (s[j] > m) m = s[j];
  double l = 0.0;
  if (m == kNegInf) {
    for (int64_t j = 0; j < n; ++j) p[j] = 0.0;
  } else {
    for (int64_t j = 0; j < n; ++j) {
      p[j] = (s[j] == kNegInf) ? 0.0 : std::exp(s[j] - m);
      l += p[j];
    }
    for (int64_t j = 0; j < n; ++j) p[j] /= l;
  }
  *m_out = m;
  *l_out = l;
}

// One output row from its score row: O = (sum_j e_j v_j) / l, LSE = m + ln l.
void attend_row(const double* s, const float* V, int64_t n_kv, int d_v, double* o, double* lse) {
  double m = kNegInf;
  for (int64_t j = 0; j < n_kv; ++j)
    if (s[j] > m) m = s[j];
  for (int c = 0; c < d_v; ++c) o[c] = 0.0;
  if (m == kNegInf) {  // no allowed key
    *lse = kNegInf;
    return;
  }
  double l = 0.0;
  for (int64_t j = 0; j < n_kv; ++j) {
    if (s[j] == kNegInf) continue;
    double e = std::exp(s[j] - m);
    l += e;
    const float* v = V + j * d_v;
    for (int c = 0; c < d_v; ++c) o[c] += e * (double)v[c];
  }
  for (int c = 0; c < d_v; ++c) o[c] /= l;
  *lse = m + std::log(l);
}

template <class F>
void parallel_for(int64_t n, int threads, F f) {
  if (threads <= 1 || n <= 1) {
    for (int64_t t = 0; t < n; ++t) f(t);
    return;
  }
  if ((int64_t)threads > n) threads = (int)n;
  std::vector<std::thread> pool;
  pool.reserve(threads);
  for (int w = 0; w < threads; ++w)
    pool.emplace_back([&, w] {
      for (int64_t t = w; t < n; t += threads) f(t);
    });
  for (auto& th : pool) th.join();
}

}  // namespace

extern "C" int oracle_scores(const float* Q, const float* K, int64_t n_q, int64_t n_kv, int d_k,
                             double scale, int causal, double* S) {
  if (n_q < 0 || n_kv < 0 || d_k <= 0 || (n_q && n_kv && (!Q || !K || !S))) return -1;
  for (int64_t i = 0; i < n_q; ++i) score_row(Q, K, i, n_q, n_kv, d_k, scale, causal, S + i * n_kv);
  return 0;
}

extern "C" int oracle_softmax_rows(const double* S, int64_t rows, int64_t cols, double* P) {
  if (rows < 0 || cols < 0 || (rows && cols && (!S || !P))) return -1;
  for (int64_t i = 0; i < rows; ++i) {
    double m, l;
    softmax_row(S + i * cols, cols, P + i * cols, &m, &l);
  }
  return 0;
}

extern "C" int oracle_softmax_naive(const double* S, int64_t rows, int64_t cols, double* P) {
  if (rows < 0 || cols < 0 || (rows && cols && (!S || !P))) return -1;
  for (int64_t i = 0; i < rows; ++i) {
    const double* s = S + i * cols;
    double* p = P + i * cols;
    double z = 0.0;
    for (int64_t j = 0; j < cols; ++j) z += std::exp(s[j]);
    for (int64_t j = 0; j < cols; ++j) p[j] = std::exp(s[j]) / z;
  }
  return 0;
}

extern "C" int oracle_sdpa_full(const float* Q, const float* K, const float* V, int64_t n_q,
                                int64_t n_kv, int d_k, int d_v, double scale, int causal,
                                double* S_out, double* P_out, double* O, double* LSE) {
  if (n_q < 0 || n_kv <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (n_q == 0) return 0;
  if (!Q || !K || !V || !O || !LSE) return -1;
  std::vector<double> S((size_t)(n_q * n_kv)), P((size_t)(n_q * n_kv));
  oracle_scores(Q, K, n_q, n_kv, d_k, scale, causal, S.data());
  for (int64_t i = 0; i < n_q; ++i) {
    double m, l;
    softmax_row(&S[(size_t)(i * n_kv)], n_kv, &P[(size_t)(i * n_kv)], &m, &l);
    for (int c = 0; c < d_v; ++c) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_kv; ++j) acc += P[(size_t)(i * n_kv + j)] * (double)V[j * d_v + c];
      O[i * d_v + c] = acc;
    }
    LSE[i] = (m == kNegInf) ? kNegInf : m + std::log(l);
  }
  if (S_out)
    for (size_t t = 0; t < S.size(); ++t) S_out[t] = S[t];
  if (P_out)
    for (size_t t = 0; t < P.size(); ++t) P_out[t] = P[t];
  return 0;
}

extern "C" int oracle_sdpa_rows(const float* Q, const float* K, const float* V, int64_t bh,
                                int64_t n_q, int64_t n_kv, int d_k, int d_v, double scale, int causal,
                                const int64_t* rows, int64_t n_rows, double* O, double* LSE,
                                int threads) {
  if (bh < 0 || n_q < 0 || n_kv <= 0 || d_k <= 0 || d_v <= 0 || n_rows < 0) return -1;
  if (!rows && n_rows != n_q) return -1;
  if (bh == 0 || n_rows == 0) return 0;
  if (!Q || !K || !V || !O || !LSE) return -1;
  for (int64_t r = 0; rows && r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= n_q) return -1;
  parallel_for(bh * n_rows, threads, [&](int64_t t) {
    int64_t b = t / n_rows, r = t % n_rows;
    int64_t i = rows ? rows[r] : r;
    std::vector<double> s((size_t)n_kv);
    const float* Qb = Q + b * n_q * d_k;
    const float* Kb = K + b * n_kv * d_k;
    const float* Vb = V + b * n_kv * d_v;
    score_row(Qb, Kb, i, n_q, n_kv, d_k, scale, causal, s.data());
    attend_row(s.data(), Vb, n_kv, d_v, O + t * d_v, LSE + t);
  });
  return 0;
}

extern "C" int oracle_decode(const float* Q, const float* K, const float* V, const int32_t* lens,
                             int64_t B, int64_t H, int64_t n_cap, int d_k, int d_v, double scale,
                             const int64_t* pairs, int64_t n_pairs, double* O, double* LSE,
                             int threads) {
  if (B < 0 || H < 0 || n_cap <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (!pairs) n_pairs = B * H;
  if (n_pairs <= 0) return 0;
  if (!Q || !K || !V || !lens || !O || !LSE) return -1;
  for (int64_t b = 0; b < B; ++b)
    if (lens[b] < 1 || lens[b] > n_cap) return -1;
  for (int64_t p = 0; pairs && p < n_pairs; ++p)
    if (pairs[p] < 0 || pairs[p] >= B * H) return -1;
  parallel_for(n_pairs, threads, [&](int64_t p) {
    int64_t bh = pairs ? pairs[p] : p;
    int64_t b = bh / H;
    int64_t n = lens[b];
    std::vector<double> s((size_t)n);
    // one query row (row 0 of a 1-row slice) against the first n keys of the cache
    score_row(Q + bh * d_k, K + bh * n_cap * d_k, 0, 1, n, d_k, scale, 0, s.data());
    attend_row(s.data(), V + bh * n_cap * d_v, n, d_v, O + p * d_v, LSE + p);
  });
  return 0;
}

extern "C" int oracle_sdpa_rows_window(const float* Q, const float* K, const float* V, int64_t bh, int64_t n_q,
                                       int64_t n_kv, int d_k, int d_v, double scale, int64_t left, int64_t right,
                                       const int64_t* rows, int64_t n_rows, double* O, double* LSE, int threads) {
  if (bh < 0 || n_q < 0 || n_kv <= 0 || d_k <= 0 || d_v <= 0 || n_rows < 0) return -1;
  if (!rows && n_rows != n_q) return -1;
  if (bh == 0 || n_rows == 0) return 0;
  if (!Q || !K || !V || !O || !LSE) return -1;
  for (int64_t r = 0; rows && r < n_rows; ++r)
    if (rows[r] < 0 || rows[r] >= n_q) return -1;
  parallel_for(bh * n_rows, threads, [&](int64_t t) {
    int64_t b = t / n_rows, r = t % n_rows;
    int64_t i = rows ? rows[r] : r;
    std::vector<double> s((size_t)n_kv);
    score_row(Q + b * n_q * d_k, K + b * n_kv * d_k, i, n_q, n_kv, d_k, scale, -1, s.data(), left, right);
    attend_row(s.data(), V + b * n_kv * d_v, n_kv, d_v, O + t * d_v, LSE + t);
  });
  return 0;
}

extern "C" int oracle_decode_gqa(const float* Q, const float* K, const float* V, const int32_t* lens, int64_t B,
                                 int64_t H_q, int64_t H_kv, int64_t n_cap, int d_k, int d_v, double scale,
                                 const int64_t* pairs, int64_t n_pairs, double* O, double* LSE, int threads) {
  if (B < 0 || H_q < 0 || H_kv <= 0 || n_cap <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (H_q % H_kv != 0) return -1;
  if (!pairs) n_pairs = B * H_q;
  if (n_pairs <= 0) return 0;
  if (!Q || !K || !V || !lens || !O || !LSE) return -1;
  for (int64_t b = 0; b < B; ++b)
    if (lens[b] < 1 || lens[b] > n_cap) return -1;
  for (int64_t p = 0; pairs && p < n_pairs; ++p)
    if (pairs[p] < 0 || pairs[p] >= B * H_q) return -1;
  const int64_t group = H_q / H_kv;  // query heads per key/value head
  parallel_for(n_pairs, threads, [&](int64_t p) {
    const int64_t bh = pairs ? pairs[p] : p;
    const int64_t b = bh / H_q, h = bh % H_q;
    const int64_t kv = b * H_kv + h / group;  // the key/value head this query head reads
    const int64_t n = lens[b];
    std::vector<double> s((size_t)n);
    score_row(Q + bh * d_k, K + kv * n_cap * d_k, 0, 1, n, d_k, scale, 0, s.data());
    attend_row(s.data(), V + kv * n_cap * d_v, n, d_v, O + p * d_v, LSE + p);
  });
  return 0;
}

extern "C" int oracle_sdpa_backward(const float* Q, const float* K, const float* V, const float* dO, int64_t bh,
                                    int64_t n_q, int64_t n_kv, int d_k, int d_v, double scale, int causal,
                                    const int64_t* q_rows, int64_t n_qr, const int64_t* k_rows, int64_t n_kr,
                                    double* dQ, double* dK, double* dV, int threads) {
  if (bh < 0 || n_q < 0 || n_kv <= 0 || d_k <= 0 || d_v <= 0) return -1;
  if (!q_rows) n_qr = n_q;
  if (!k_rows) n_kr = n_kv;
  if (n_qr < 0 || n_kr < 0) return -1;
  if (bh == 0 || n_q == 0) return 0;
  if (!Q || !K || !V || !dO) return -1;
  for (int64_t r = 0; q_rows && r < n_qr; ++r)
    if (q_rows[r] < 0 || q_rows[r] >= n_q) return -1;
  for (int64_t r = 0; k_rows && r < n_kr; ++r)
    if (k_rows[r] < 0 || k_rows[r] >= n_kv) return -1;
  // where each query / key row lands in the outputs (-1: not requested)
  std::vector<int64_t> q_slot((size_t)n_q, -1), k_slot((size_t)n_kv, -1);
  for (int64_t r = 0; r < n_qr; ++r) q_slot[(size_t)(q_rows ? q_rows[r] : r)] = r;
  for (int64_t r = 0; r < n_kr; ++r) k_slot[(size_t)(k_rows ? k_rows[r] : r)] = r;
  parallel_for(bh, threads, [&](int64_t b) {
    const float* Qb = Q + b * n_q * d_k;
    const float* Kb = K + b * n_kv * d_k;
    const float* Vb = V + b * n_kv * d_v;
    const float* dOb = dO + b * n_q * d_v;
    double* dQb = dQ ? dQ + b * n_qr * d_k : nullptr;
    double* dKb = dK ? dK + b * n_kr * d_k : nullptr;
    double* dVb = dV ? dV + b * n_kr * d_v : nullptr;
    if (dQb)
      for (int64_t t = 0; t < n_qr * d_k; ++t) dQb[t] = 0.0;
    if (dKb)
      for (int64_t t = 0; t < n_kr * d_k; ++t) dKb[t] = 0.0;
    if (dVb)
      for (int64_t t = 0; t < n_kr * d_v; ++t) dVb[t] = 0.0;
    std::vector<double> s((size_t)n_kv), p((size_t)n_kv), dp((size_t)n_kv);
    for (int64_t i = 0; i < n_q; ++i) {
      // row i of P = softmax(S): the forward definition
      score_row(Qb, Kb, i, n_q, n_kv, d_k, scale, causal, s.data());
      double m, l;
      softmax_row(s.data(), n_kv, p.data(), &m, &l);
      if (m == kNegInf) continue;  // no allowed key: no gradient flows through this row
      // row i of dP = dO V^T, and the softmax Jacobian's row term sum_k P_ik dP_ik
      const float* dOi = dOb + i * d_v;
      double rowdot = 0.0;
      for (int64_t j = 0; j < n_kv; ++j) {
        double acc = 0.0;
        const float* vj = Vb + j * d_v;
        for (int c = 0; c < d_v; ++c) acc += (double)dOi[c] * (double)vj[c];
        dp[(size_t)j] = acc;
        rowdot += p[(size_t)j] * acc;
      }
      const int64_t qi = q_slot[(size_t)i];
      for (int64_t j = 0; j < n_kv; ++j) {
        const double pij = p[(size_t)j];
        if (pij == 0.0) continue;
        const double dsij = pij * (dp[(size_t)j] - rowdot);
        if (dQb && qi >= 0) {  // dQ_i += scale dS_ij K_j
          const float* kj = Kb + j * d_k;
          for (int c = 0; c < d_k; ++c) dQb[qi * d_k + c] += scale * dsij * (double)kj[c];
        }
        const int64_t kj_slot = k_slot[(size_t)j];
        if (kj_slot < 0) continue;
        if (dVb)  // dV_j += P_ij dO_i
          for (int c = 0; c < d_v; ++c) dVb[kj_slot * d_v + c] += pij * (double)dOi[c];
        if (dKb) {  // dK_j += scale dS_ij Q_i
          const float* qi_row = Qb + i * d_k;
          for (int c = 0; c < d_k; ++c) dKb[kj_slot * d_k + c] += scale * dsij * (double)qi_row[c];
        }
      }
    }
  });
  return 0;
}
