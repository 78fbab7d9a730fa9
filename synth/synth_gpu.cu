/*
 * Seeded synthetic input generator, device build (see synth_core.h).  Same
 * element-for-element definition as synth_cpu.c, so the bytes it writes equal
 * the CPU build's (checked by a GPU test on sampled ranges).  Exported with C
 * linkage for ctypes; device pointers in, asynchronous on the given stream.
 *
 * Build: nvcc -gencode arch=compute_100a,code=sm_100a -fmad=false -shared
 */
#include <cuda_runtime.h>
#include <stdint.h>

#include "synth_core.h"

#define EXPORT extern "C" __attribute__((visibility("default")))

namespace {

__global__ void fill_kernel(uint64_t key, int dist, double p0, double p1, uint64_t offset, uint64_t n,
                            int out_fmt, void* out) {
  for (uint64_t t = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; t < n;
       t += (uint64_t)gridDim.x * blockDim.x) {
    double v = dist == 0 ? p0 + p1 * synth_normal(key, offset + t) : synth_uniform(key, offset + t, p0, p1);
    if (out_fmt == 2) {
      ((double*)out)[t] = v;
    } else if (out_fmt == 0) {
      ((float*)out)[t] = __double2float_rn(v);
    } else {
      ((uint16_t*)out)[t] = synth_f32_to_bf16(__double2float_rn(v));
    }
  }
}

/* one warp per 128-block: 4 values per lane */
__global__ void fill_fp8_kernel(uint64_t key, double std, uint64_t nblocks, uint8_t* q, float* s) {
  const int lane = threadIdx.x & 31;
  uint64_t warp = (blockIdx.x * (uint64_t)blockDim.x + threadIdx.x) >> 5;
  uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  for (uint64_t b = warp; b < nblocks; b += nwarps) {
    float v[4];
    float amax = 0.0f;
    for (int i = 0; i < 4; ++i) {
      v[i] = __double2float_rn(std * synth_normal(key, b * 128 + lane * 4 + i));
      amax = fmaxf(amax, fabsf(v[i]));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    float sc = synth_fp8_block_scale(amax);
    if (lane == 0) s[b] = sc;
    uint32_t packed = 0;
    for (int i = 0; i < 4; ++i) packed |= (uint32_t)synth_fp8_encode(v[i], sc) << (8 * i);
    ((uint32_t*)(q + b * 128))[lane] = packed;
  }
}

/* one warp per 32-block: 1 value per lane, nibbles paired through a shuffle */
__global__ void fill_mxfp4_kernel(uint64_t key, double std, uint64_t nblocks, uint32_t spread, uint8_t* q, uint8_t* e) {
  const int lane = threadIdx.x & 31;
  uint64_t warp = (blockIdx.x * (uint64_t)blockDim.x + threadIdx.x) >> 5;
  uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
  for (uint64_t b = warp; b < nblocks; b += nwarps) {
    float v = __double2float_rn(ldexp(std, -(int)synth_mx_shift(b, spread)) * synth_normal(key, b * 32 + lane));
    float amax = fabsf(v);
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    uint8_t sb = synth_mx_scale_byte(amax);
    if (lane == 0) e[b] = sb;
    uint32_t c = synth_mx_encode(v, sb);
    uint32_t hi = __shfl_down_sync(0xffffffffu, c, 1);
    if ((lane & 1) == 0) q[b * 16 + (lane >> 1)] = (uint8_t)(c | (hi << 4));
  }
}

int grid_for(uint64_t work, int threads) {
  uint64_t g = (work + threads - 1) / threads;
  if (g > 148ull * 64) g = 148ull * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

EXPORT int synth_gpu_fill(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, int dist, double p0,
                          double p1, uint64_t offset, uint64_t n, int out_fmt, void* out, void* stream) {
  if (n == 0) return 0;
  uint64_t key = synth_key(seed, layer, kind, expert);
  fill_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(key, dist, p0, p1, offset, n, out_fmt, out);
  return (int)cudaGetLastError();
}

EXPORT int synth_gpu_fill_fp8(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, double std,
                              uint64_t rows, uint64_t cols, uint8_t* q, float* s, void* stream) {
  uint64_t nb = rows * (cols / 128);
  if (nb == 0) return 0;
  uint64_t key = synth_key(seed, layer, kind, expert);
  fill_fp8_kernel<<<grid_for(nb * 32, 256), 256, 0, (cudaStream_t)stream>>>(key, std, nb, q, s);
  return (int)cudaGetLastError();
}

EXPORT int synth_gpu_fill_mxfp4(uint64_t seed, uint32_t layer, uint32_t kind, uint32_t expert, double std,
                                uint64_t rows, uint64_t cols, uint32_t spread, uint8_t* q, uint8_t* e, void* stream) {
  uint64_t nb = rows * (cols / 32);
  if (nb == 0) return 0;
  uint64_t key = synth_key(seed, layer, kind, expert);
  fill_mxfp4_kernel<<<grid_for(nb * 32, 256), 256, 0, (cudaStream_t)stream>>>(key, std, nb, spread, q, e);
  return (int)cudaGetLastError();
}
