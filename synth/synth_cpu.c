/*
 * Seeded synthetic input generator, CPU build (see synth_core.h for the
 * definitions).  Exported with C linkage for ctypes; every function fills
 * caller-owned host memory.  OpenMP splits the element range; each element
 * depends only on (seed, tensor tag, index), so the output does not depend on
 * the thread count.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -fPIC -shared
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#include "synth_core.h"

#define EXPORT __attribute__((visibility("default")))

enum { OUT_F32 = 0, OUT_BF16 = 1, OUT_F64 = 2 };

/* dist 0: p0 + p1 * N(0,1);  dist 1: U[p0, p1) */
static inline double draw(uint64_t key, uint64_t i, int dist, double p0, double p1) {
  if (dist == 0) return p0 + p1 * synth_normal(key, i);
  return synth_uniform(key, i, p0, p1);
}

EXPORT void synth_fill(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, int dist,
                       double p0, double p1, uint64_t offset, uint64_t n, int out_fmt, void* out) {
  uint64_t key = synth_key(seed, layer, kind, expert);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < (int64_t)n; ++t) {
    double v = draw(key, offset + (uint64_t)t, dist, p0, p1);
    if (out_fmt == OUT_F64) {
      ((double*)out)[t] = v;
    } else if (out_fmt == OUT_F32) {
      ((float*)out)[t] = (float)v;
    } else {
      ((uint16_t*)out)[t] = synth_f32_to_bf16((float)v);
    }
  }
}

/* FP8 e4m3 weights [rows][cols] with fp32 scales [rows][cols/128] */
EXPORT void synth_quant_fp8(const float* w, uint64_t rows, uint64_t cols, uint8_t* q, float* s) {
  uint64_t nb = cols / 128;
#pragma omp parallel for schedule(static)
  for (int64_t rb = 0; rb < (int64_t)(rows * nb); ++rb) {
    const float* src = w + (uint64_t)rb * 128;
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
      float a = src[i] < 0.0f ? -src[i] : src[i];
      if (a > amax) amax = a;
    }
    float sc = synth_fp8_block_scale(amax);
    s[rb] = sc;
    for (int i = 0; i < 128; ++i) q[(uint64_t)rb * 128 + i] = synth_fp8_encode(src[i], sc);
  }
}

/* MXFP4 weights [rows][cols/2] (even element in the low nibble) with e8m0
 * scales [rows][cols/32] */
EXPORT void synth_quant_mxfp4(const float* w, uint64_t rows, uint64_t cols, uint8_t* q, uint8_t* e) {
  uint64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t rb = 0; rb < (int64_t)(rows * nb); ++rb) {
    const float* src = w + (uint64_t)rb * 32;
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
      float a = src[i] < 0.0f ? -src[i] : src[i];
      if (a > amax) amax = a;
    }
    uint8_t sb = synth_mx_scale_byte(amax);
    e[rb] = sb;
    for (int i = 0; i < 16; ++i) {
      uint8_t lo = synth_mx_encode(src[2 * i], sb);
      uint8_t hi = synth_mx_encode(src[2 * i + 1], sb);
      q[(uint64_t)rb * 16 + i] = (uint8_t)(lo | (hi << 4));
    }
  }
}

/* normal weights std * N(0,1), rounded to fp32, then quantised, without
 * holding the fp32 tensor: one 128- or 32-block at a time. */
EXPORT void synth_fill_fp8(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, double std,
                           uint64_t rows, uint64_t cols, uint8_t* q, float* s) {
  uint64_t key = synth_key(seed, layer, kind, expert);
  uint64_t nb = cols / 128;
#pragma omp parallel for schedule(static)
  for (int64_t rb = 0; rb < (int64_t)(rows * nb); ++rb) {
    float buf[128];
    float amax = 0.0f;
    for (int i = 0; i < 128; ++i) {
      buf[i] = (float)(std * synth_normal(key, (uint64_t)rb * 128 + i));
      float a = buf[i] < 0.0f ? -buf[i] : buf[i];
      if (a > amax) amax = a;
    }
    float sc = synth_fp8_block_scale(amax);
    s[rb] = sc;
    for (int i = 0; i < 128; ++i) q[(uint64_t)rb * 128 + i] = synth_fp8_encode(buf[i], sc);
  }
}

EXPORT void synth_fill_mxfp4(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, double std,
                             uint64_t rows, uint64_t cols, uint32_t spread, uint8_t* q, uint8_t* e) {
  uint64_t key = synth_key(seed, layer, kind, expert);
  uint64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t rb = 0; rb < (int64_t)(rows * nb); ++rb) {
    float buf[32];
    float amax = 0.0f;
    for (int i = 0; i < 32; ++i) {
      buf[i] = (float)(ldexp(std, -(int)synth_mx_shift((uint64_t)rb, spread)) * synth_normal(key, (uint64_t)rb * 32 + i));
      float a = buf[i] < 0.0f ? -buf[i] : buf[i];
      if (a > amax) amax = a;
    }
    uint8_t sb = synth_mx_scale_byte(amax);
    e[rb] = sb;
    for (int i = 0; i < 16; ++i) {
      uint8_t lo = synth_mx_encode(buf[2 * i], sb);
      uint8_t hi = synth_mx_encode(buf[2 * i + 1], sb);
      q[(uint64_t)rb * 16 + i] = (uint8_t)(lo | (hi << 4));
    }
  }
}

EXPORT double synth_ln_probe(double x) { return synth_ln(x); }
EXPORT uint32_t synth_abi_version(void) { return 1u; }
