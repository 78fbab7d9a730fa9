/*
 * Seeded synthetic input generator: the arithmetic shared by the CPU build
 * (synth_cpu.c) and the device build (synth_gpu.cu) of the SAME generator.
 *
 * This module only makes test/benchmark inputs.  It holds none of the layer's
 * arithmetic: no norm, no mix, no router, no expert math.  It does hold the
 * weight ENCODERS (fp32 -> bf16 / FP8-e4m3 1x128 / MXFP4), because a
 * synthetic "checkpoint" must be quantised before the layer can read it; the
 * oracle carries its own, independently written encoder and a CPU test checks
 * that both produce the same bytes.
 *
 * Both builds must produce bit-identical values, so everything here uses only
 * integer operations and IEEE-754 +, -, *, / and sqrt in double (correctly
 * rounded on both sides); callers compile with FMA contraction disabled
 * (gcc -ffp-contract=off, nvcc -fmad=false).  No libm transcendental is used:
 * the logarithm below is evaluated from its atanh series.
 *
 * Definitions
 *   mix64(z)       SplitMix64 output function (Steele, Lea, Flood, "Fast
 *                  splittable pseudorandom number generators", OOPSLA 2014;
 *                  constants of the public-domain splitmix64.c by S. Vigna).
 *   bits(key, c)   the c-th output of a SplitMix64 stream whose state starts
 *                  at key: mix64(key + (c + 1) * GAMMA).  Counter-based, so any
 *                  element can be generated on its own.
 *   normal(key,i)  Marsaglia polar method (Marsaglia & Bray 1964), attempt j of
 *                  sample i drawing counters 64*i + 2j and 64*i + 2j + 1;
 *                  returns v1 * sqrt(-2 ln s / s) of the first accepted pair.
 */
#ifndef SYNTH_CORE_H
#define SYNTH_CORE_H

#include <stdint.h>

#ifdef __CUDACC__
#define SYNTH_FN __host__ __device__ static inline
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ull

/* tensor kinds, part of the per-tensor stream tag */
enum {
  SYNTH_HC_IN = 1,
  SYNTH_MIX_W = 2,
  SYNTH_NORM_W = 3,
  SYNTH_ROUTER_W = 4,
  SYNTH_ROUTER_BIAS = 5,
  SYNTH_GATE = 6,
  SYNTH_UP = 7,
  SYNTH_DOWN = 8,
  SYNTH_ATTN_X = 9,     /* the attention sublayer's pending state (within-layer boundary) */
  SYNTH_ATTN_POST = 10,
  SYNTH_ATTN_COMB = 11,
  SYNTH_ATTN_Y = 12
};

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* stream key of one tensor: seed, layer, kind and expert slot */
SYNTH_FN uint64_t synth_key(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert) {
  uint64_t tag = ((uint64_t)layer << 40) | ((uint64_t)kind << 32) | (uint64_t)expert;
  return synth_mix64(synth_mix64(seed * SYNTH_GAMMA + 0x5851F42D4C957F2Dull) ^ synth_mix64(tag + 1));
}

SYNTH_FN uint64_t synth_bits(uint64_t key, uint64_t ctr) {
  return synth_mix64(key + (ctr + 1) * SYNTH_GAMMA);
}

/* uniform in [0, 1) with 53 random bits (exact) */
SYNTH_FN double synth_u53(uint64_t b) {
  return (double)(b >> 11) * (1.0 / 9007199254740992.0);
}

SYNTH_FN uint64_t synth_d2u(double x) {
  union { double d; uint64_t u; } v;
  v.d = x;
  return v.u;
}
SYNTH_FN double synth_u2d(uint64_t x) {
  union { double d; uint64_t u; } v;
  v.u = x;
  return v.d;
}
SYNTH_FN uint32_t synth_f2u(float x) {
  union { float f; uint32_t u; } v;
  v.f = x;
  return v.u;
}
SYNTH_FN float synth_u2f(uint32_t x) {
  union { float f; uint32_t u; } v;
  v.u = x;
  return v.f;
}

/* natural log of a positive normal double, from
 *   ln(m * 2^e) = e ln2 + 2 atanh((m - 1) / (m + 1)),  m in [sqrt(1/2), sqrt(2))
 * with the atanh series summed to t^23 (|t| < 0.172, truncation < 1e-18). */
SYNTH_FN double synth_ln(double x) {
  uint64_t u = synth_d2u(x);
  int e = (int)((u >> 52) & 0x7FF) - 1023;
  double m = synth_u2d((u & 0x000FFFFFFFFFFFFFull) | 0x3FF0000000000000ull); /* [1,2) */
  if (m > 1.4142135623730951) {
    m = m * 0.5;
    e = e + 1;
  }
  double t = (m - 1.0) / (m + 1.0);
  double t2 = t * t;
  double p = 1.0 / 23.0;
  p = p * t2 + 1.0 / 21.0;
  p = p * t2 + 1.0 / 19.0;
  p = p * t2 + 1.0 / 17.0;
  p = p * t2 + 1.0 / 15.0;
  p = p * t2 + 1.0 / 13.0;
  p = p * t2 + 1.0 / 11.0;
  p = p * t2 + 1.0 / 9.0;
  p = p * t2 + 1.0 / 7.0;
  p = p * t2 + 1.0 / 5.0;
  p = p * t2 + 1.0 / 3.0;
  p = p * t2 + 1.0;
  return (double)e * 0.6931471805599453 + 2.0 * t * p;
}

/* standard normal sample i of stream key (double) */
SYNTH_FN double synth_normal(uint64_t key, uint64_t i) {
  for (uint64_t j = 0; j < 32; ++j) {
    double v1 = 2.0 * synth_u53(synth_bits(key, 64 * i + 2 * j)) - 1.0;
    double v2 = 2.0 * synth_u53(synth_bits(key, 64 * i + 2 * j + 1)) - 1.0;
    double s = v1 * v1 + v2 * v2;
    if (s < 1.0 && s > 0.0) return v1 * sqrt(-2.0 * synth_ln(s) / s);
  }
  return 0.0;
}

/* uniform sample i of stream key on [lo, hi) (double) */
SYNTH_FN double synth_uniform(uint64_t key, uint64_t i, double lo, double hi) {
  return lo + (hi - lo) * synth_u53(synth_bits(key, i));
}

/* fp32 -> bf16 bits, round to nearest even (NaN kept quiet) */
SYNTH_FN uint16_t synth_f32_to_bf16(float f) {
  uint32_t u = synth_f2u(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* |f| -> e4m3fn magnitude code (7 bits), round to nearest even, saturating at
 * 448 (code 0x7E).  e4m3fn: 4 exponent bits (bias 7), 3 mantissa bits,
 * subnormal step 2^-9, no infinities. */
SYNTH_FN uint32_t synth_e4m3_mag(float a) {
  uint32_t u = synth_f2u(a) & 0x7FFFFFFFu;
  if (u >= 0x43E00000u) return 0x7Eu; /* >= 448 */
  int e = (int)(u >> 23) - 127;
  if (e < -6) {
    /* subnormal range: value = k * 2^-9 with k in [0, 8]; k = rne(a * 2^9) */
    double k = (double)a * 512.0; /* exact */
    double fl = (double)(int64_t)k;
    double fr = k - fl;
    int64_t q = (int64_t)fl;
    if (fr > 0.5 || (fr == 0.5 && (q & 1))) q += 1;
    return (uint32_t)q; /* q == 8 is the smallest normal, code 0x08 */
  }
  /* normal: keep 3 mantissa bits, RNE on the 20 dropped bits */
  uint32_t mant = u & 0x7FFFFFu;
  uint32_t keep = mant >> 20;
  uint32_t rest = mant & 0xFFFFFu;
  uint32_t code = ((uint32_t)(e + 7) << 3) | keep;
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) code += 1;
  if (code > 0x7Eu) code = 0x7Eu;
  return code;
}

/* |f| -> e2m1 magnitude code (3 bits), round to nearest even, saturating at 6.
 * e2m1 magnitudes by code: 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
SYNTH_FN uint32_t synth_e2m1_mag(float a) {
  if (a <= 0.25f) return 0;
  if (a < 0.75f) return 1;
  if (a <= 1.25f) return 2;
  if (a < 1.75f) return 3;
  if (a <= 2.5f) return 4;
  if (a < 3.5f) return 5;
  if (a <= 5.0f) return 6;
  return 7;
}

/* FP8 1x128 block encoder: s = amax / 448 (1 if amax == 0), q = e4m3(w / s) */
SYNTH_FN float synth_fp8_block_scale(float amax) {
  return amax > 0.0f ? amax / 448.0f : 1.0f;
}
SYNTH_FN uint8_t synth_fp8_encode(float w, float s) {
  float v = w / s;
  uint32_t sign = (synth_f2u(v) >> 31) << 7;
  return (uint8_t)(sign | synth_e4m3_mag(v < 0.0f ? -v : v));
}

/* Spread of block magnitudes within a row, for the MXFP4 generator: block b
 * of an expert's blocks is drawn at std * 2^-k with k = synth_mx_shift(b,
 * spread) in [0, spread] (0 when spread is 0), so that a row's block scales
 * span up to 2^spread.  Real checkpoints hold blocks far below their row's
 * largest; the default workloads use spread 0. */
SYNTH_FN uint32_t synth_mx_shift(uint64_t b, uint32_t spread) {
  if (spread == 0u) return 0u;
  uint64_t h = (b + 1u) * 0x9E3779B97F4A7C15ull;
  return (uint32_t)((h >> 40) % (uint64_t)(spread + 1u));
}

/* MXFP4 32-block encoder (OCP MX v1.0 shared-exponent rule):
 * X = floor(log2 amax) - 2 (e2m1's largest exponent), stored as the e8m0 byte
 * X + 127 clamped to [0, 254]; amax == 0 stores byte 0. */
SYNTH_FN uint8_t synth_mx_scale_byte(float amax) {
  if (!(amax > 0.0f)) return 0;
  uint32_t u = synth_f2u(amax);
  int e = (int)(u >> 23) - 127;
  if ((u >> 23) == 0) { /* subnormal amax: locate its leading bit */
    uint32_t m = u & 0x7FFFFFu;
    e = -127;
    while (m < 0x800000u) {
      m <<= 1;
      e -= 1;
    }
    e += 1;
  }
  int b = e - 2 + 127;
  if (b < 0) b = 0;
  if (b > 254) b = 254;
  return (uint8_t)b;
}
SYNTH_FN uint8_t synth_mx_encode(float w, uint8_t scale_byte) {
  /* w * 2^-(X): computed in double so that it is exact, then rounded to fp32
   * (exact unless far below the block amax, where only the sign survives). */
  double p = synth_u2d((uint64_t)(1023 - ((int)scale_byte - 127)) << 52);
  float v = (float)((double)w * p);
  uint32_t sign = (synth_f2u(v) >> 31) << 3;
  return (uint8_t)(sign | synth_e2m1_mag(v < 0.0f ? -v : v));
}

#endif
