// Router select that allocates nothing: a standalone variant of the fused
// kernel's router stage (logits over all experts, sqrt(softplus) scores,
// selection bias, canonical top-k, normalised and scaled weights).
//
// Why it exists: some callers cannot allocate device memory at the moment
// they need a routing decision.  A serving engine that reserves all device
// memory up front and hands out nothing during decode, or code running
// between two captured graph segments that must not touch the allocator,
// has no plan to borrow scratch from and cannot make one.  This entry point
// keeps its scratch (per-split partial logits and one arrival counter) in a
// fixed static device array instead of allocated memory.
//
// Scratch contract:
//   - the partial logits need no initial value: every call writes every
//     element it reads;
//   - the arrival counter must start at zero.  It is zero from static
//     initialisation at module load, and every call's last block sets it
//     back to zero before it returns;
//   - calls that overlap in time on the same device (two streams, or two
//     host threads without ordering) share the scratch and race: order them
//     on one stream or with events.
#pragma once
#include <atomic>

#include "common.cuh"

namespace mono {

constexpr int kRtMaxR = 8, kRtMaxE = 1024, kRtMaxK = 16;
constexpr int kRtSplit = 8;            // contraction splits, one grid column each
constexpr int kRtThreads = 256;        // 8 warps, lane = expert within a group of 32

struct RtScratch {
  float part[kRtSplit][kRtMaxR][kRtMaxE];   // partial logits, one slab per split
  unsigned int arrivals;                    // blocks done with this call (0 between calls)
};

// 256-byte aligned, 256 KB + one counter: the whole scratch of every call on
// this device
static __device__ __align__(256) RtScratch g_route_scratch;

// Block (g, s): experts [32 g, 32 g + 32), contraction slice s of kRtSplit.
// The block that arrives last sums the splits in order and selects.
__global__ void __launch_bounds__(kRtThreads) route_noalloc_kernel(int R, int H, int E, int K, const void* n, int n_bf16,
                                                                   const float* __restrict__ router_w,
                                                                   const float* __restrict__ bias, float route_scale,
                                                                   float denom_clamp, int* idx, float* wout,
                                                                   RtScratch* sc) {
  __shared__ float red[kRtThreads / 32][kRtMaxR][32];
  __shared__ int last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 32 + lane, s = blockIdx.y;
  const int h0 = (int)((long long)s * H / kRtSplit), h1 = (int)((long long)(s + 1) * H / kRtSplit);
  float acc[kRtMaxR];
#pragma unroll
  for (int r = 0; r < kRtMaxR; ++r) acc[r] = 0.f;
  if (e < E) {
#pragma unroll 4
    for (int h = h0 + warp; h < h1; h += kRtThreads / 32) {
      const float wv = __ldg(router_w + (size_t)h * E + e);
#pragma unroll
      for (int r = 0; r < kRtMaxR; ++r) {
        if (r < R) {
          const float nv = n_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(n)[(size_t)r * H + h])
                                  : reinterpret_cast<const float*>(n)[(size_t)r * H + h];
          acc[r] = fmaf(nv, wv, acc[r]);
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRtMaxR; ++r) red[warp][r][lane] = acc[r];
  __syncthreads();
  if (warp == 0 && e < E) {
    for (int r = 0; r < R; ++r) {
      float t = 0.f;
      for (int q = 0; q < kRtThreads / 32; ++q) t += red[q][r][lane];
      sc->part[s][r][e] = t;
    }
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int total = gridDim.x * gridDim.y;
    last = atomicAdd(&sc->arrivals, 1u) == total - 1u;
  }
  __syncthreads();
  if (!last) return;
  __threadfence();
  // the last block: logits = sum of the splits in order, then one warp per
  // row: scores, canonical (selection desc, index asc) top-k, weights
  for (int r = warp; r < R; r += kRtThreads / 32) {
    float lg[kRtMaxE / 32], bs[kRtMaxE / 32];
#pragma unroll
    for (int q = 0; q < kRtMaxE / 32; ++q) {
      const int ee = lane + 32 * q;
      lg[q] = 0.f;
      bs[q] = 0.f;
      if (ee < E) {
        for (int ss = 0; ss < kRtSplit; ++ss) lg[q] += __ldcg(&sc->part[ss][r][ee]);
        bs[q] = __ldg(bias + ee);
      }
    }
    select_row<kRtMaxE / 32>(
        lg, bs, E, K, denom_clamp, route_scale, [&](int j, int e) { idx[r * K + j] = e; },
        [&](int j, float wv) { wout[r * K + j] = wv; });
  }
  __syncthreads();
  if (threadIdx.x == 0) atomicExch(&sc->arrivals, 0u);   // ready for the next call
}

}  // namespace mono

namespace {

constexpr int kRtMaxDevices = 64;
std::atomic<void*> g_route_scratch_ptr[kRtMaxDevices] = {};   // per device, from the first call on it

}  // namespace

extern "C" int mono_ffn_route_noalloc(int rows, int hidden, int n_routed, int top_k, const void* n, int n_bf16,
                                      const float* router_w, const float* router_bias, float route_scale,
                                      float denom_clamp, int* idx, float* w, void* stream) {
  using namespace mono;
  std::string why;
  if (rows < 0) why += "rows must be >= 0\n";
  if (rows > kRtMaxR) why += "rows " + std::to_string(rows) + " above the scratch limit " + std::to_string(kRtMaxR) + "\n";
  if (hidden <= 0) why += "hidden must be > 0\n";
  if (n_routed <= 0 || n_routed > kRtMaxE)
    why += "n_routed " + std::to_string(n_routed) + " outside 1.." + std::to_string(kRtMaxE) + " (the scratch limit)\n";
  if (top_k <= 0 || top_k > kRtMaxK || top_k > n_routed)
    why += "top_k " + std::to_string(top_k) + " outside 1..min(" + std::to_string(kRtMaxK) + ", n_routed)\n";
  if (rows > 0 && (!n || !router_w || !router_bias || !idx || !w)) why += "NULL tensor pointer\n";
  if (!why.empty()) return fail(nullptr, MONO_ERR_INVALID_ARG, "route_noalloc: " + why);
  if (rows == 0) return MONO_OK;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "route_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kRtMaxDevices) return fail(nullptr, MONO_ERR_INVALID_ARG, "route_noalloc: device id above 63");
  void* sc = g_route_scratch_ptr[dev].load();
  if (!sc) {
    // first call on this device: the static scratch's device address (this
    // may load the module, so make the first call outside stream capture)
    e = cudaGetSymbolAddress(&sc, g_route_scratch);
    if (e != cudaSuccess) return cuda_fail(nullptr, e, "route_noalloc: cudaGetSymbolAddress");
    g_route_scratch_ptr[dev].store(sc);
  }
  const dim3 grid((unsigned)((n_routed + 31) / 32), (unsigned)kRtSplit);
  route_noalloc_kernel<<<grid, kRtThreads, 0, (cudaStream_t)stream>>>(rows, hidden, n_routed, top_k, n, n_bf16, router_w,
                                                                       router_bias, route_scale, denom_clamp, idx, w,
                                                                       reinterpret_cast<RtScratch*>(sc));
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(nullptr, e, "route_noalloc: launch");
  return MONO_OK;
}
