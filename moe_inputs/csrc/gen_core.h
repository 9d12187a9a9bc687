/*
 * gen_core.h -- the seeded, counter-based input generator shared by the host
 * (C++) and device (CUDA) builds of libmoeinputs.
 *
 * This file is INPUT GENERATION ONLY. It holds none of the MoE layer's
 * arithmetic: it turns (seed, stream id, element index) into a number with a
 * stated distribution, identically on the CPU and on the GPU, so that both the
 * CPU oracle and the CUDA path can be fed the same synthetic tensors.
 *
 * Building blocks (all published methods, written from their definitions):
 *   - Philox-4x32-10 counter-based generator: Salmon, Moraes, Dror, Shaw,
 *     "Parallel random numbers: as easy as 1, 2, 3", SC'11.  Multipliers
 *     0xD2511F53 / 0xCD9E8D57, Weyl key increments 0x9E3779B9 / 0xBB67AE85.
 *   - Box-Muller transform (Box & Muller, 1958): two uniforms -> two N(0,1).
 *   - ln(m) for m in [sqrt(1/2), sqrt(2)) by the series
 *       ln m = 2 * (s + s^3/3 + s^5/5 + ...),  s = (m-1)/(m+1)
 *     (the atanh series), after exact power-of-two range reduction.
 *   - sin/cos of 2*pi*u by exact quadrant reduction and Taylor series on
 *     [0, pi/2).
 * Every floating-point step is an IEEE-754 double add/mul/div/sqrt in a fixed
 * order with no fused multiply-add, so host and device produce bit-identical
 * doubles; those are then rounded to fp32 (round to nearest even) and, for
 * bf16 tensors, from fp32 to bf16 (round to nearest even).
 *
 * Element index i of a tensor with (seed, stream) uses Philox block i/4 with
 * counter (lo32(i/4), hi32(i/4), 0, 0) and key (lo32(seed), stream).  Word
 * w = i%4 of that block is the uniform source for element i; normals use the
 * pair (2*(w/2), 2*(w/2)+1) and take the cosine branch for even w and the
 * sine branch for odd w.
 */
#ifndef MOE_INPUTS_GEN_CORE_H
#define MOE_INPUTS_GEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define MI_HD __host__ __device__ __forceinline__
#else
#define MI_HD static inline
#endif

/* Fixed-order IEEE double arithmetic, no contraction on either side. */
#if defined(__CUDA_ARCH__)
#define MI_ADD(a, b) __dadd_rn((a), (b))
#define MI_SUB(a, b) __dsub_rn((a), (b))
#define MI_MUL(a, b) __dmul_rn((a), (b))
#define MI_DIV(a, b) __ddiv_rn((a), (b))
#define MI_SQRT(a) __dsqrt_rn((a))
#else
#include <math.h>
#define MI_ADD(a, b) ((a) + (b))
#define MI_SUB(a, b) ((a) - (b))
#define MI_MUL(a, b) ((a) * (b))
#define MI_DIV(a, b) ((a) / (b))
#define MI_SQRT(a) sqrt((a))
#endif

typedef struct {
  uint32_t v[4];
} mi_u32x4;

MI_HD uint32_t mi_mulhi32(uint32_t a, uint32_t b) {
  return (uint32_t)(((uint64_t)a * (uint64_t)b) >> 32);
}

/* Philox-4x32 with 10 rounds on counter c under key k. */
MI_HD mi_u32x4 mi_philox4x32_10(mi_u32x4 c, uint32_t k0, uint32_t k1) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  for (int r = 0; r < 10; ++r) {
    uint32_t hi0 = mi_mulhi32(M0, c.v[0]);
    uint32_t lo0 = M0 * c.v[0];
    uint32_t hi1 = mi_mulhi32(M1, c.v[2]);
    uint32_t lo1 = M1 * c.v[2];
    mi_u32x4 n;
    n.v[0] = hi1 ^ c.v[1] ^ k0;
    n.v[1] = lo1;
    n.v[2] = hi0 ^ c.v[3] ^ k1;
    n.v[3] = lo0;
    c = n;
    k0 += W0;
    k1 += W1;
  }
  return c;
}

MI_HD mi_u32x4 mi_block(uint64_t seed, uint32_t stream, uint64_t block) {
  mi_u32x4 c;
  c.v[0] = (uint32_t)block;
  c.v[1] = (uint32_t)(block >> 32);
  c.v[2] = 0u;
  c.v[3] = 0u;
  return mi_philox4x32_10(c, (uint32_t)seed, stream);
}

/* Uniform in the open interval (0, 1): (w + 1/2) / 2^32, exact in double. */
MI_HD double mi_u01_open(uint32_t w) {
  return MI_MUL(MI_ADD((double)w, 0.5), 2.3283064365386962890625e-10);
}

/* Uniform in [0, 1): w / 2^32, exact in double. */
MI_HD double mi_u01_closed_open(uint32_t w) {
  return MI_MUL((double)w, 2.3283064365386962890625e-10);
}

/* Natural log of u in (0, 1), u >= 2^-33 (always a normal double here). */
MI_HD double mi_ln(double u) {
  /* u = m * 2^e with m in [1, 2): read the exponent field directly. */
  union {
    double d;
    uint64_t b;
  } cv;
  cv.d = u;
  int e = (int)((cv.b >> 52) & 0x7FF) - 1023;
  cv.b = (cv.b & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull;
  double m = cv.d;
  if (m > 1.4142135623730951) { /* keep m in [sqrt(1/2), sqrt(2)) */
    m = MI_MUL(m, 0.5);
    e += 1;
  }
  double s = MI_DIV(MI_SUB(m, 1.0), MI_ADD(m, 1.0));
  double s2 = MI_MUL(s, s);
  /* Horner in s^2 over the odd reciprocals 1/1, 1/3, ..., 1/25. */
  double p = MI_DIV(1.0, 25.0);
  for (int n = 23; n >= 1; n -= 2) p = MI_ADD(MI_DIV(1.0, (double)n), MI_MUL(s2, p));
  double lnm = MI_MUL(2.0, MI_MUL(s, p));
  return MI_ADD(MI_MUL((double)e, 0.6931471805599453), lnm);
}

/* sin and cos of 2*pi*u for u in [0, 1). */
MI_HD void mi_sincos_2pi(double u, double* sn, double* cs) {
  double v = MI_MUL(u, 4.0); /* exact */
  int q = (int)v;            /* quadrant 0..3 */
  double r = MI_SUB(v, (double)q); /* exact, in [0, 1) */
  double x = MI_MUL(r, 1.5707963267948966);
  double x2 = MI_MUL(x, x);
  /* Taylor: sin x = x(1 - x^2/(2*3)(1 - x^2/(4*5)(1 - ...))), to x^23. */
  double ps = 1.0;
  for (int n = 22; n >= 2; n -= 2) ps = MI_SUB(1.0, MI_MUL(MI_DIV(x2, (double)(n * (n + 1))), ps));
  double sx = MI_MUL(x, ps);
  /* cos x = 1 - x^2/(1*2)(1 - x^2/(3*4)(1 - ...)), to x^24. */
  double pc = 1.0;
  for (int n = 23; n >= 1; n -= 2) pc = MI_SUB(1.0, MI_MUL(MI_DIV(x2, (double)(n * (n + 1))), pc));
  double cx = pc;
  switch (q) {
    case 0: *sn = sx; *cs = cx; break;
    case 1: *sn = cx; *cs = -sx; break;
    case 2: *sn = -sx; *cs = -cx; break;
    default: *sn = -cx; *cs = sx; break;
  }
}

/* Standard normal for element index i (Box-Muller on a word pair). */
MI_HD double mi_normal(uint64_t seed, uint32_t stream, uint64_t i) {
  mi_u32x4 b = mi_block(seed, stream, i >> 2);
  uint32_t w = (uint32_t)(i & 3u);
  uint32_t p = w >> 1;
  double u1 = mi_u01_open(b.v[2 * p]);
  double u2 = mi_u01_closed_open(b.v[2 * p + 1]);
  double rad = MI_SQRT(MI_MUL(-2.0, mi_ln(u1)));
  double sn, cs;
  mi_sincos_2pi(u2, &sn, &cs);
  return (w & 1u) ? MI_MUL(rad, sn) : MI_MUL(rad, cs);
}

/* Uniform in (lo, hi) for element index i. */
MI_HD double mi_uniform(uint64_t seed, uint32_t stream, uint64_t i, double lo, double hi) {
  mi_u32x4 b = mi_block(seed, stream, i >> 2);
  double u = mi_u01_open(b.v[i & 3u]);
  return MI_ADD(lo, MI_MUL(MI_SUB(hi, lo), u));
}

/* fp32 -> bf16 bits, round to nearest even (inputs here are finite). */
MI_HD uint16_t mi_f32_to_bf16_bits(float f) {
  union {
    float f;
    uint32_t u;
  } cv;
  cv.f = f;
  uint32_t u = cv.u;
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif /* MOE_INPUTS_GEN_CORE_H */
