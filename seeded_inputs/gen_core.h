/*
 * Seeded, counter-based input generation shared by the CPU (oracle side) and
 * the GPU (device buffers for the CUDA path).  Test and benchmark plumbing
 * only: nothing here computes any part of attention.
 *
 * Every value is a pure function of (seed, stream, counter):
 *   - SplitMix64 (Steele, Lea, Flood, "Fast Splittable Pseudorandom Number
 *     Generators", OOPSLA 2014).  The n-th output of a SplitMix64 generator
 *     whose state starts at s is mix(s + (n+1)*gamma).  A stream's starting
 *     state is output number `stream` of a generator seeded with `seed`.
 *   - Normal deviates: Box-Muller (1958).  One 64-bit draw gives the pair
 *     (u1, u2); element 2i takes r*cos(theta), element 2i+1 takes
 *     r*sin(theta), r = sqrt(-2 ln u1), theta = 2*pi*u2.
 *   - Uniform deviates: the top 24 bits of the draw, scaled to [0, 1).
 *
 * Bit-identical host/device results: ln, sin and cos are evaluated here with
 * IEEE add, multiply, divide and square root only (all correctly rounded in
 * both gcc/x86-64 SSE2 and CUDA *_rn intrinsics), in a fixed order, with no
 * fused multiply-add.  ln uses the series ln m = 2 atanh((m-1)/(m+1)) after an
 * exact binary reduction of m to [sqrt(1/2), sqrt(2)]; sin and cos use their
 * Taylor series in nested form after an exact quadrant reduction of the
 * angle, which is held as a 24-bit fraction of a full turn.  Truncation error
 * is below 1e-16, far below what the float32/bf16 rounding keeps.
 */
#ifndef SEEDED_INPUTS_GEN_CORE_H
#define SEEDED_INPUTS_GEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define GEN_FN static __host__ __device__ __forceinline__
#else
#define GEN_FN static inline
#include <string.h>
#endif

#define GEN_SM64_GAMMA 0x9E3779B97F4A7C15ULL

GEN_FN double g_add(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dadd_rn(a, b);
#else
  return a + b;
#endif
}
GEN_FN double g_sub(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dsub_rn(a, b);
#else
  return a - b;
#endif
}
GEN_FN double g_mul(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dmul_rn(a, b);
#else
  return a * b;
#endif
}
GEN_FN double g_div(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}
GEN_FN double g_sqrt(double a) {
#if defined(__CUDA_ARCH__)
  return __dsqrt_rn(a);
#else
  return __builtin_sqrt(a);
#endif
}
GEN_FN float g_to_f32(double a) {
#if defined(__CUDA_ARCH__)
  return __double2float_rn(a);
#else
  return (float)a;
#endif
}
GEN_FN uint32_t g_f32_bits(float f) {
#if defined(__CUDA_ARCH__)
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return u;
#endif
}
GEN_FN int g_clz32(uint32_t x) {
#if defined(__CUDA_ARCH__)
  return __clz((int)x);
#else
  return __builtin_clz(x);
#endif
}
/* 2^e for -1022 <= e <= 1023, built from its bit pattern (exact). */
GEN_FN double g_pow2(int e) {
  uint64_t bits = (uint64_t)(e + 1023) << 52;
#if defined(__CUDA_ARCH__)
  return __longlong_as_double((long long)bits);
#else
  double d;
  memcpy(&d, &bits, sizeof d);
  return d;
#endif
}

/* SplitMix64 output finaliser. */
GEN_FN uint64_t gen_sm64_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}
/* Starting state of stream `stream` under `seed`. */
GEN_FN uint64_t gen_stream_state(uint64_t seed, uint64_t stream) {
  return gen_sm64_mix(seed + (stream + 1ULL) * GEN_SM64_GAMMA);
}
/* Draw number `ctr` of a stream. */
GEN_FN uint64_t gen_draw(uint64_t state, uint64_t ctr) {
  return gen_sm64_mix(state + (ctr + 1ULL) * GEN_SM64_GAMMA);
}

/* ln(k * 2^-24) for 1 <= k <= 2^24. */
GEN_FN double gen_ln_k24(uint32_t k) {
  int e = 31 - g_clz32(k);                  /* k = m * 2^e, m in [1, 2) */
  double m = g_mul((double)k, g_pow2(-e));  /* exact */
  if (m > 1.4142135623730951) {             /* reduce to [sqrt(1/2), sqrt(2)] */
    m = g_mul(m, 0.5);
    e += 1;
  }
  double t = g_div(g_sub(m, 1.0), g_add(m, 1.0)); /* |t| <= 0.1716 */
  double t2 = g_mul(t, t);
  /* sum_{i=0}^{13} t2^i / (2i+1), Horner from the top term */
  double acc = g_div(1.0, 27.0);
  for (int i = 12; i >= 0; --i) acc = g_add(g_mul(acc, t2), g_div(1.0, (double)(2 * i + 1)));
  double ln_m = g_mul(g_mul(2.0, t), acc);
  const double LN2 = 0x1.62E42FEFA39EFp-1;
  return g_add(g_mul((double)(e - 24), LN2), ln_m);
}

/* cos and sin of 2*pi*k2*2^-24 for 0 <= k2 < 2^24. */
GEN_FN void gen_cossin_turn24(uint32_t k2, double* c_out, double* s_out) {
  uint32_t quadrant = k2 >> 22;
  double f = g_mul((double)(k2 & 0x3FFFFFu), 0x1p-24);  /* [0, 1/4), exact */
  const double TWO_PI = 0x1.921FB54442D18p+2;
  double x = g_mul(f, TWO_PI);                           /* [0, pi/2) */
  double x2 = g_mul(x, x);
  /* sin x = x (1 - x^2/(2*3) (1 - x^2/(4*5) (1 - ...))), cos x = 1 - x^2/(1*2) (1 - x^2/(3*4) (...)) */
  double s = 1.0, c = 1.0;
  for (int i = 13; i >= 1; --i) {
    s = g_sub(1.0, g_mul(g_div(x2, (double)((2 * i) * (2 * i + 1))), s));
    c = g_sub(1.0, g_mul(g_div(x2, (double)((2 * i - 1) * (2 * i))), c));
  }
  s = g_mul(x, s);
  double cr, sr;
  switch (quadrant) {
    case 0: cr = c; sr = s; break;
    case 1: cr = -s; sr = c; break;
    case 2: cr = -c; sr = -s; break;
    default: cr = s; sr = -c; break;
  }
  *c_out = cr;
  *s_out = sr;
}

/* Element `idx` of a standard normal stream (Box-Muller pairs). */
GEN_FN double gen_normal_at(uint64_t state, uint64_t idx) {
  uint64_t z = gen_draw(state, idx >> 1);
  uint32_t k1 = (uint32_t)(z >> 40) + 1u;          /* u1 = k1 * 2^-24 in (0, 1] */
  uint32_t k2 = (uint32_t)(z >> 16) & 0xFFFFFFu;   /* u2 = k2 * 2^-24 in [0, 1) */
  double r = g_sqrt(g_mul(-2.0, gen_ln_k24(k1)));
  double c, s;
  gen_cossin_turn24(k2, &c, &s);
  return g_mul(r, (idx & 1ULL) ? s : c);
}

/* Element `idx` of a uniform [0, 1) stream. */
GEN_FN double gen_unit_at(uint64_t state, uint64_t idx) {
  uint64_t z = gen_draw(state, idx);
  return g_mul((double)(uint32_t)(z >> 40), 0x1p-24);
}

/* float32 -> bfloat16 bits, round to nearest even; NaN stays a quiet NaN. */
GEN_FN uint16_t gen_f32_to_bf16(float f) {
  uint32_t u = g_f32_bits(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x0040u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Distribution kinds. */
enum { GEN_NORMAL = 0, GEN_UNIFORM = 1 };

/* One value as float32: normal -> a + b*N(0,1); uniform -> a + (b-a)*U[0,1). */
GEN_FN float gen_value_f32(int kind, uint64_t state, uint64_t idx, double a, double b) {
  if (kind == GEN_NORMAL) return g_to_f32(g_add(a, g_mul(b, gen_normal_at(state, idx))));
  return g_to_f32(g_add(a, g_mul(g_sub(b, a), gen_unit_at(state, idx))));
}

#endif
