// Device code shared by the two persistent "mono" kernels (one launch runs the
// whole FFN half-layer): constants, the per-CTA control block, bounded waits,
// the prologue (hyper-connection mix, collapse + weighted RMSNorm, router
// logits, top-k and work lists) and the tail (routed + shared sum, expand).
//
// Warp roles inside a CTA (384 threads, both kernels):
//   warps 0-7    compute: prologue, then the expert phase of the kernel, tail
//   warp  8      producer: 1-D TMA bulk copies of packed weight chunks into
//                the shared-memory ring (mbarrier complete_tx)
//   warp  9      tensor-core issuer (tcgen05.mma) in the tensor-core kernel
//   warps 10-11  control: Sinkhorn, the canonical top-k, the expert lists
//
// Grid-wide dependencies are counters in global memory that are never reset
// between launches: each counter a kernel waits on takes one arrival (a
// release-add) from every CTA in every launch, so at a launch's start it
// holds the completion counter's value b, and a CTA waits with acquire loads
// until it reaches b + grid (modulo 2^32, so wrap-safe).  Every wait is
// bounded by the plan's timeout; on expiry the CTA records an error word,
// raises the abort flag and runs the rest of its control flow without waiting
// (so every named barrier is still reached), then returns.
#pragma once
#include <cuda.h>

#include <type_traits>

#include "ptx.cuh"

namespace mono {

constexpr int kS = 4;         // hyper-connection streams
constexpr int kMixC = 24;     // 2S + S*S
constexpr int kMixP = 25;     // mix columns + the square sum
constexpr int kMaxR = 8;
constexpr int kMaxK = 16;
constexpr int kMaxU = kMaxR * kMaxK;
constexpr int kMaxE = 1024;
constexpr int kCW = 8;        // compute warps (also the items of a CUDA-core ring stage)
constexpr int kProdWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kCtlWarp0 = 10;
constexpr int kCtlWarps = 2;
constexpr int kThreads = 12 * 32;                      // 384: 12 warps leave 168 registers a thread
constexpr int kPreThreads = (kCW + kCtlWarps) * 32;    // compute + control
// named barriers: prologue (compute + control), compute, control, epilogue
// warps 0-3, routing hand-over (compute + control), end (epilogue warps + the
// issuer warp)
constexpr int kBarPre = 1, kBarCons = 2, kBarCtl = 3, kBarEpi = 4, kBarRoute = 5, kBarEnd = 6, kBarTop = 7;
constexpr int kMaxAcc = 4;         // accumulator buffers in tensor memory
constexpr int kRingGuard = 4096;   // bytes after the ring that a tensor-core tile may read past its stage

enum WType { W_F32 = 0, W_BF16 = 1, W_FP8 = 2, W_FP4 = 3 };

struct SyncBlock {   // one per layer slot, 64 bytes
  uint32_t epoch, cnt_mix, cnt_logit, cnt_act, cnt_done, cnt_y, cnt_a, cnt_mix2, pad[8];
};
struct ErrBlock {
  uint32_t abort, code, stage, cta, layer, pad[11];
};

struct Taps {
  float *mix, *pre, *post, *comb, *n, *logits;
  int* idx;
  float *w, *y, *x;
};

struct Params {
  int H, I, E, K, R, G;
  int layer, first, last;
  int dense;            // no router: every slot is a slice of one dense MLP, weight 1
  int mx8;              // MXFP4 experts with MXFP8 activations (one e4m3 term per row, N = 8)
  int mix_ctas;
  int hc_bf16, norm_bf16, round_bf16;
  float rms_eps, pre_eps, post_mult, route_scale, denom_clamp;
  int sink_iters;
  // residual streams
  const void* x_prev;   // first: this layer's X (hc_in); else the residual streams before the
                        // pending expand (the previous layer's X, or the attention sublayer's input)
  void* xbuf;           // this layer's X when not first (written by the mix CTAs)
  void* hc_out;         // written when last
  const float* pend_post; // the pending expand (not first): post [R][4] and comb [R][16] fp32,
  const float* pend_comb; // and y [R][H] (fp32, or bf16 when pend_y_bf16), of the previous layer
  const void* pend_y;     // or of the attention sublayer
  int pend_y_bf16;
  float* pend_out;      // this layer's pending state (when not last)
  // packed weights
  const float* mix_w;
  const void* norm_w;
  const float* router_t;   // [E][H]
  const float* bias;
  // CUDA-core kernel: gu [E+1][I][gu_nk][gate|up][gu_rc], dn [E+1][H][dn_nk][dn_rc]
  //   (row chunks of kc elements with their block scales);
  // tensor-core kernel: gu [E+1][I/128][H/8][16][gate|up][8][8],
  //   dn [E+1][H/128][I/8][16][8][8] (blocks of 128 output rows made of bf16
  //   core matrices of 8 rows x 8 contraction elements)
  const uint8_t* gu;
  const uint8_t* dn;
  int gu_kc, gu_nk, gu_rc;
  int dn_kc, dn_nk, dn_rc;
  long long gu_estride, dn_estride;
  // scratch
  float* mix_part;   // [R*25][G] output-major partials of the mix
  float* mix_tot;    // [R*25] the mix totals (each summed by one CTA)
  float* logits;     // [R][E]
  float* act;        // [R][K+1][I]
  void* abuf;        // [R][H] collapsed rows a (bf16 when rounded, else fp32), one h-slice per CTA
  float* sq_part;    // [R][G] per-CTA partial sums of a^2
  float* yp;         // tensor-core kernel: [R][K+1][H] weighted expert outputs
  uint32_t* xready;  // tensor-core kernel: [R*K+1] finished gate/up blocks per expert entry (0 between steps)
  const float* gsc;  // tensor-core FP8 kernel: [E+1][I/128][H/128][gate 128 | up 128] fp32 block scales;
                     // MXFP4: [E+1][I/128][H/128][gate | up] 512-byte e8m0 scale chunks
  const float* dsc;  // tensor-core FP8 kernel: [E+1][H/128][I/128][128] fp32 block scales;
                     // MXFP4: [E+1][H/128][I/128] 512-byte e8m0 scale chunks
  CUtensorMap tm_gu; // MXFP4 tensor-core kernel: 2-D maps of the packed gate/up and down codes,
  CUtensorMap tm_dn; // rows of 128 e2m1 codes, unpacked into 16-byte slots, 128-byte swizzle
  int n_xready;
  int n_xready_all;   // the plan's entries (max rows x top_k + 1): all cleared each launch
  uint8_t* actb;     // tensor-core kernel: [R*K+1][I/8][16][8] bf16 down-projection B operands
  float* gpart;      // tensor-core kernel: [G][4][128][16] partial gate|up tiles of split blocks
  float* dpart;      // tensor-core kernel: [G][2][128][16] partial down tiles
  uint32_t* gcnt;    // tensor-core kernel: [R*K+2][I/128] arrivals per split gate/up block (0 between launches)
  uint32_t* dcnt;    // tensor-core kernel: [R*K+2][H/128] arrivals per split down block
  SyncBlock* sync;
  ErrBlock* err;
  Taps taps;
  int nst, slot_bytes, regA_bytes, ymax;
  unsigned long long timeout_ns;
  const int* row_slot;  // [R] int32: row r is padding when row_slot[r] < 0 (NULL: every row live)
  int fault_cta;      // tests: this CTA withholds its arrival at fault_stage (-1: none)
  int fault_stage;    // MONO_STAGE_* of the withheld arrival
  unsigned jitter_ns; // tests: every publishing thread first sleeps up to this long (0: off)
  unsigned long long* trace;   // optional [G][kTracePoints] globaltimer stamps
};

constexpr int kTracePoints = 32;
// stage timestamps (one writer per point and CTA)
__device__ __forceinline__ void trace(const Params& p, int point, bool who = true) {
  if (p.trace && who) p.trace[blockIdx.x * kTracePoints + point] = globaltimer();
}

// Before a grid-visible arrival (a counter other CTAs wait on) at `stage`:
// in the race-detection mode the publishing thread first sleeps a pseudo-
// random time hash(CTA, epoch, point) % jitter_ns, so that arrival orders
// change from step to step; returns false when this CTA is the one told to
// withhold its arrival at this stage (fault injection of the tests).
__device__ __forceinline__ bool may_publish(const Params& p, uint32_t epoch, int stage, uint32_t point) {
  if (p.jitter_ns) {
    uint32_t h = blockIdx.x * 0x9E3779B1u ^ (epoch + 0x7F4A7C15u) * 0x85EBCA77u ^ point * 0xC2B2AE3Du;
    h ^= h >> 15;
    h *= 0x2C1B3C6Du;
    h ^= h >> 12;
    __nanosleep(h % p.jitter_ns);
  }
  return !((int)blockIdx.x == p.fault_cta && stage == p.fault_stage);
}

// per-CTA control block in shared memory
struct Ctl {
  volatile int dead;
  volatile int lists_ready;
  uint32_t epoch;
  uint32_t live;                // bit r: row r is a live row (not padding)
  volatile int nu;              // unique routed experts (control warps' copy)
  int nu_comp;                  // the compute warps' agreed copy
  float smix[kMaxR][kMixP];     // mix partial totals, then the scaled mix
  float pre[kMaxR][kS], post[kMaxR][kS], comb[kMaxR][kS * kS];
  float inv[kMaxR];
  float sq[kCW][kMaxR];
  float sq2[kCW][kMaxR];
  uint32_t bm[kMaxE / 32];      // selected-expert bitmap
  int nu_ctl;
  int idx[kMaxR][kMaxK];
  float wt[kMaxR][kMaxK];
  int ulist[kMaxU];
  uint32_t umask[kMaxU];
  signed char uslot[kMaxU][kMaxR];
  float red[kPreThreads * 2];
  // tensor-core kernel
  uint32_t tmem_base;
  volatile int n_ready;         // n is in shared memory (B operand of gate/up)
  uint64_t accfull[kMaxAcc], accempty[kMaxAcc], drain;
  uint64_t bfull;               // the down projection's B operand has landed
  volatile int bcast;           // epilogue: "this CTA completes the block"
  // FP8 tensor-core kernel: inverse power-of-two scale of each row of n, and
  // the epilogue warps' per-row maxima of a block's activations
  float nsc[kMaxR];
  float amax[4][kMaxR];
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// dynamic shared memory layout
struct SmemLayout {
  size_t bars, ctl, ys, regA, ring, total;
  __host__ __device__ SmemLayout(int nst, int slot_bytes, int regA_bytes, int ymax) {
    bars = 0;
    ctl = align_up(bars + 2 * 8 * (size_t)nst, 128);
    ys = align_up(ctl + sizeof(Ctl), 128);
    regA = align_up(ys + sizeof(float) * kMaxR * (size_t)ymax, 128);
    ring = align_up(regA + (size_t)regA_bytes, 1024);
    total = ring + (size_t)nst * slot_bytes + kRingGuard;
  }
};

// Rows of the launch that are live (bit r), from the optional row slots: a
// padding row (slot < 0) reads as zero, selects no expert and writes nothing.
__device__ __forceinline__ uint32_t live_rows(const Params& p) {
  uint32_t m = 0u;
  for (int r = 0; r < p.R; ++r)
    if (!p.row_slot || __ldg(p.row_slot + r) >= 0) m |= 1u << r;
  return m;
}

// ------------------------------------------------------------ bounded waits --

__device__ __forceinline__ void record_error(const Params& p, Ctl* c, uint32_t code, uint32_t stage) {
  if (atomicCAS(&p.err->code, 0u, code) == 0u) {
    p.err->stage = stage;
    p.err->cta = blockIdx.x;
    p.err->layer = p.layer;
  }
  atomicExch(&p.err->abort, 1u);
  c->dead = 1;
}

// wait until *cnt >= target (wrap-safe); false when dead or timed out
__device__ bool wait_count(const Params& p, Ctl* c, const uint32_t* cnt, uint32_t target, uint32_t stage) {
  volatile int* dead = &c->dead;
  uint64_t t0 = globaltimer();
  uint32_t ns = 32, it = 0;
  while (true) {
    if (*dead) return false;
    uint32_t v = ld_acquire(cnt);
    if ((int32_t)(v - target) >= 0) return true;
    // the abort word and the clock every eighth poll, so that a poll is one
    // round trip (an acquire load orders the loads after it)
    if ((++it & 7u) == 0u) {
      if (ld_relaxed(&p.err->abort)) {
        c->dead = 1;
        return false;
      }
      if (globaltimer() - t0 > p.timeout_ns) {
        record_error(p, c, 7u, stage);   // MONO_ERR_DEVICE_TIMEOUT (negated on the host)
        return false;
      }
    }
    __nanosleep(ns);
    if (ns < 128) ns <<= 1;
  }
}

__device__ bool wait_bar(const Params& p, Ctl* c, uint64_t* bar, uint32_t parity) {
  volatile int* dead = &c->dead;
  if (mbar_try(bar, parity)) return true;   // waits in hardware, wakes on the phase
  uint64_t t0 = globaltimer();
  while (true) {
    if (*dead) return false;
    if (mbar_try(bar, parity)) return true;
    if (globaltimer() - t0 > 2 * p.timeout_ns) {   // downstream of the grid-wide waits
      record_error(p, c, 7u, 5u);
      return false;
    }
  }
}

__device__ bool wait_flag(const Params& p, Ctl* c, volatile int* flag) {
  volatile int* dead = &c->dead;
  uint64_t t0 = globaltimer();
  while (true) {
    if (*flag) return true;
    if (*dead) return false;
    if (globaltimer() - t0 > 2 * p.timeout_ns) {   // downstream of the grid-wide waits
      record_error(p, c, 7u, 3u);
      return false;
    }
    __nanosleep(64);
  }
}

// --------------------------------------------------------------- helpers --

__device__ __forceinline__ float load_x(const void* base, size_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return reinterpret_cast<const float*>(base)[i];
}
__device__ __forceinline__ float load_x_cg(const void* base, size_t i, int bf16) {
  if (bf16) {
    unsigned short b = __ldcg(reinterpret_cast<const unsigned short*>(base) + i);
    return __uint_as_float((uint32_t)b << 16);
  }
  return __ldcg(reinterpret_cast<const float*>(base) + i);
}
__device__ __forceinline__ void store_x(void* base, size_t i, float v, int bf16) {
  if (bf16) reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(base)[i] = v;
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// ordered key of a float for a max-reduction (larger float -> larger key)
__device__ __forceinline__ uint32_t ord_key(float x) {
  x = x + 0.0f;   // -0 -> +0
  uint32_t b = __float_as_uint(x);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <int WT> struct WFmt;
template <> struct WFmt<W_F32> { static constexpr int EPU = 4; };
template <> struct WFmt<W_BF16> { static constexpr int EPU = 8; };
template <> struct WFmt<W_FP8> { static constexpr int EPU = 16; };
template <> struct WFmt<W_FP4> { static constexpr int EPU = 32; };

// scale of weight unit u (16 bytes) of a row chunk that holds kc elements
template <int WT>
__device__ __forceinline__ float unit_scale(const uint8_t* chunk, int kc, int u) {
  if (WT == W_FP8) return reinterpret_cast<const float*>(chunk + kc)[u >> 3];       // 8 units per 128
  if (WT == W_FP4) {
    uint32_t e = chunk[kc / 2 + u];
    return e ? __uint_as_float(e << 23) : __uint_as_float(0x00400000u);             // 2^(e-127)
  }
  return 1.0f;
}

// load NE activation values (elements k .. k+NE-1) of a row as floats
template <int NE, bool BF>
__device__ __forceinline__ void load_vec(const void* row, int k, float* f) {
  if (BF) {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(row) + k;
    if (NE % 8 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 8; ++i) {
        uint4 v = reinterpret_cast<const uint4*>(src)[i];
        f[8 * i + 0] = bf16lo(v.x); f[8 * i + 1] = bf16hi(v.x);
        f[8 * i + 2] = bf16lo(v.y); f[8 * i + 3] = bf16hi(v.y);
        f[8 * i + 4] = bf16lo(v.z); f[8 * i + 5] = bf16hi(v.z);
        f[8 * i + 6] = bf16lo(v.w); f[8 * i + 7] = bf16hi(v.w);
      }
    } else if (NE % 2 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 2; ++i) {
        uint32_t v = reinterpret_cast<const uint32_t*>(src)[i];
        f[2 * i] = bf16lo(v);
        f[2 * i + 1] = bf16hi(v);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NE; ++i) f[i] = __uint_as_float((uint32_t)src[i] << 16);
    }
  } else {
    const float* src = reinterpret_cast<const float*>(row) + k;
    if (NE % 4 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 4; ++i) {
        float4 v = reinterpret_cast<const float4*>(src)[i];
        f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
      }
    } else if (NE % 2 == 0) {
#pragma unroll
      for (int i = 0; i < NE / 2; ++i) {
        float2 v = reinterpret_cast<const float2*>(src)[i];
        f[2 * i] = v.x; f[2 * i + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NE; ++i) f[i] = src[i];
    }
  }
}

// 16-byte units in the code part of a row chunk of kc elements
template <int WT> __device__ __forceinline__ int units_of(int kc) {
  return WT == W_F32 ? kc / 4 : WT == W_BF16 ? kc / 8 : WT == W_FP8 ? kc / 16 : kc / 32;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 8 consecutive activation values (bf16 or fp32 storage) at element i
__device__ __forceinline__ void load_hc8(const void* base, size_t i, int bf16, float* f) {
  if (bf16) {
    const uint4 v = __ldcg(reinterpret_cast<const uint4*>(reinterpret_cast<const uint16_t*>(base) + i));
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
  } else {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i) + 1);
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(lo)) |
         ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(hi)) << 16);
}
// 8 values to shared memory: bf16 (exact for values already rounded) or fp32
__device__ __forceinline__ void store8(uint8_t* base, size_t i, bool bf, const float* f) {
  if (bf) {
    uint4 v;
    v.x = pack_bf16x2(f[0], f[1]); v.y = pack_bf16x2(f[2], f[3]);
    v.z = pack_bf16x2(f[4], f[5]); v.w = pack_bf16x2(f[6], f[7]);
    reinterpret_cast<uint4*>(base + i * 2)[0] = v;
  } else {
    reinterpret_cast<float4*>(base + i * 4)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(base + i * 4)[1] = make_float4(f[4], f[5], f[6], f[7]);
  }
}
__device__ __forceinline__ void load8(const uint8_t* base, size_t i, bool bf, float* f) {
  if (bf) {
    const uint4 v = reinterpret_cast<const uint4*>(base + i * 2)[0];
    f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
    f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
  } else {
    const float4 a = reinterpret_cast<const float4*>(base + i * 4)[0];
    const float4 b = reinterpret_cast<const float4*>(base + i * 4)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w; f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
}

// The router select of one row by one warp, from each expert's logit and
// bias (lane l holds experts l + 32 q, q < NQ; experts >= E are ignored):
// score = sqrt(softplus(logit)) in fp32, sel = score + bias, the canonical
// top-k by (sel desc, index asc) through warp max / min reductions, then
// weight = score / max(sum, clamp) * scale with each op rounded to fp32.
// put_idx(j, e) runs on lane 0 for selection j; after a warp sync,
// put_w(j, w) runs on lane j < K.  Shared by the fused kernels' top-k and
// the allocation-free router select, so the two cannot drift apart.
template <int NQ, class FI, class FW>
__device__ __forceinline__ void select_row(const float (&lg)[NQ], const float (&bs)[NQ], int E, int K, float denom_clamp,
                                           float route_scale, FI put_idx, FW put_w) {
  const int lane = threadIdx.x & 31;
  float score[NQ];
  uint32_t key[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = lane + 32 * q;
    score[q] = 0.f;
    key[q] = 0u;
    if (e < E) {
      const float sp = fmaxf(lg[q], 0.f) + log1pf(expf(-fabsf(lg[q])));
      score[q] = sqrtf(sp);
      key[q] = ord_key(score[q] + bs[q]);
    }
  }
  uint32_t taken = 0u;
  float ssum = 0.f, wsel = 0.f;
  for (int j = 0; j < K; ++j) {
    uint32_t bk = 0u;
    int be = 0x7FFFFFFF;
    float bsc = 0.f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      if (!((taken >> q) & 1u) && key[q] > bk) {
        bk = key[q];
        be = lane + 32 * q;
        bsc = score[q];
      }
    }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
    const int we = (int)__reduce_min_sync(0xffffffffu, (uint32_t)(bk == wk ? be : 0x7FFFFFFF));
    const int wl = we & 31;
    if (we < E && wl == lane) taken |= 1u << (we >> 5);
    const float ws = __shfl_sync(0xffffffffu, bsc, wl);
    if (lane == j) wsel = ws;   // lane j keeps the j-th raw score
    if (lane == 0) put_idx(j, we < E ? we : 0);
    ssum += ws;   // selection order, fp32
  }
  __syncwarp();
  if (lane < K) {
    const float den = fmaxf(ssum, denom_clamp);
    put_w(lane, __fmul_rn(__fdiv_rn(wsel, den), route_scale));
  }
  __syncwarp();
}

// The fused kernels' top-k of row r: every CTA's logits and the bias, then
// select_row into the control block.  dry: run the same code without storing
// anything (it is then warm in the SM's instruction cache when the real call
// comes); not inlined, so that the dry and the real call share one copy.
template <int NQ>
__device__ __noinline__ void topk_row(const Params& p, Ctl* c, int r, bool dry) {
  const int lane = threadIdx.x & 31;
  const int E = p.E;
  // every load first (a store in between would order them one by one)
  float lg[NQ], bs[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = lane + 32 * q;
    lg[q] = (e < E && !c->dead) ? __ldcg(p.logits + (size_t)r * E + e) : 0.f;
    bs[q] = e < E ? __ldg(p.bias + e) : 0.f;
  }
  if (blockIdx.x == 0 && p.taps.logits && !dry) {
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (lane + 32 * q < E) p.taps.logits[(size_t)r * E + lane + 32 * q] = lg[q];
  }
  trace(p, 26, r == 0 && lane == 0 && !dry);
  select_row<NQ>(
      lg, bs, E, p.K, p.denom_clamp, p.route_scale,
      [&](int j, int e) {
        if (!dry) c->idx[r][j] = e;
      },
      [&](int j, float w) {
        if (dry) return;
        c->wt[r][j] = w;
        if (blockIdx.x == 0) {
          if (p.taps.idx) p.taps.idx[r * p.K + j] = c->idx[r][j];
          if (p.taps.w) p.taps.w[r * p.K + j] = w;
        }
      });
}

// A dense layer's "routing" of row r (one warp): every routed slot, in slot
// order, with weight 1 (the shared slot joins as always).
__device__ __forceinline__ void dense_row(const Params& p, Ctl* c, int r) {
  const int lane = threadIdx.x & 31;
  if (lane < p.K) {
    c->idx[r][lane] = lane;
    c->wt[r][lane] = 1.0f;
    if (blockIdx.x == 0) {
      if (p.taps.idx) p.taps.idx[r * p.K + lane] = lane;
      if (p.taps.w) p.taps.w[r * p.K + lane] = 1.0f;
    }
  }
  __syncwarp();
}

// the top-k of row r with the lane layout that fits E
__device__ __forceinline__ void topk_dispatch(const Params& p, Ctl* c, int r, bool dry) {
  const int E = p.E;
  if (E <= 32) topk_row<1>(p, c, r, dry);
  else if (E <= 64) topk_row<2>(p, c, r, dry);
  else if (E <= 128) topk_row<4>(p, c, r, dry);
  else if (E <= 256) topk_row<8>(p, c, r, dry);
  else if (E <= 512) topk_row<16>(p, c, r, dry);
  else topk_row<32>(p, c, r, dry);
}

// ------------------------------------------------------------ work walkers --

// The stage sequence of one CTA.  Producer and consumers run the same walker;
// a stage is (phase, expert slot, first item, items, chunk index).
enum Phase { PH_SGU = 0, PH_RGU = 1, PH_DN = 2 };

struct Walk {
  // shared expert gate/up: channels [c0, c1)
  __device__ static void sgu_range(const Params& p, int& c0, int& c1) {
    c0 = (int)(blockIdx.x * (uint32_t)p.I / (uint32_t)p.G);
    c1 = (int)((blockIdx.x + 1) * (uint32_t)p.I / (uint32_t)p.G);
  }
  // routed gate/up over the unique-expert list: global channels [g0, g1)
  __device__ static void rgu_range(const Params& p, int nu, long long& g0, long long& g1) {
    long long n = (long long)nu * p.I;
    g0 = (long long)blockIdx.x * n / p.G;
    g1 = (long long)(blockIdx.x + 1) * n / p.G;
  }
  // down: output channels [h0, h1) of every expert
  __device__ static void dn_range(const Params& p, int& h0, int& h1) {
    h0 = (int)(blockIdx.x * (uint32_t)p.H / (uint32_t)p.G);
    h1 = (int)((blockIdx.x + 1) * (uint32_t)p.H / (uint32_t)p.G);
  }
};

// ============================================================== prologue ==
// Thread numbering of the prologue group (compute warps 0-7 and control warps
// 10-11): 0 .. kPreThreads-1.
__device__ __forceinline__ int pre_tid() {
  const int t = threadIdx.x;
  return t < kCW * 32 ? t : t - (kCtlWarp0 - kCW) * 32;
}

// Shared-memory offsets of the prologue's staging areas inside regA: the
// CTA's slice of mix_w [S][nh][24], its slice of the residual streams
// [R][S][nh] (kept until the collapse has used it), then room for the mix
// partials of every CTA.
struct PreLayout {
  int h0, h1, nh;
  size_t ws, xs, parts;
  __device__ PreLayout(const Params& p) {
    Walk::dn_range(p, h0, h1);
    nh = h1 - h0;
    ws = 0;
    xs = ws + (size_t)kS * nh * kMixC * 4;
    parts = align_up(xs + (size_t)p.R * kS * nh * 4, 16);
  }
};

// A2 (every CTA, on the h-range it also owns in the tail): materialise this
// layer's residual streams from the previous layer's pending post/comb expand
// (or read hc_in), then the partial mix products and square sums.  A3: wait
// for every CTA's partials, reduce them in one fixed order in every CTA, and
// derive rho, mix, pre and post.  Loads are issued all at once (cp.async /
// unrolled) so that each stage costs one memory round trip.
__device__ void prologue_mix(const Params& p, Ctl* c, uint8_t* regA, uint32_t ep1) {
  const int R = p.R, H = p.H, G = p.G;
  const int ptid = pre_tid(), pwarp = ptid >> 5, lane = threadIdx.x & 31;
  const int nout = R * kMixP;
  const PreLayout L(p);
  const int h0 = L.h0, nh = L.nh;
  float* ws = reinterpret_cast<float*>(regA + L.ws);   // [S][nh][24] slice of mix_w
  float* xs = reinterpret_cast<float*>(regA + L.xs);   // [R][S][nh]
  {
    // mix_w rows s * H + h0 .. + nh are contiguous: 16-byte asynchronous copies
    const int seg4 = nh * (kMixC / 4);
    for (int i = ptid; i < kS * seg4; i += kPreThreads) {
      const int sgm = i / seg4, j = i % seg4;
      cp_async16(reinterpret_cast<float4*>(ws) + i, reinterpret_cast<const float4*>(p.mix_w + ((size_t)sgm * H + h0) * kMixC) + j);
    }
    cp_async_commit();
    const float* ppost = p.pend_post;
    const float* pcomb = p.pend_comb;
    const int nx = R * kS * nh;
    constexpr int kXU = 4;   // elements per thread in flight
    for (int i0 = ptid; i0 < nx; i0 += kXU * kPreThreads) {
      float v[kXU];
#pragma unroll
      for (int u = 0; u < kXU; ++u) {
        const int i = i0 + u * kPreThreads;
        v[u] = 0.f;
        if (i < nx) {
          const int r = i / (kS * nh), sg = (i / nh) % kS, h = h0 + i % nh;
          if (!((c->live >> r) & 1u)) {
            v[u] = 0.f;   // padding row: its input is ignored
          } else if (p.first) {
            v[u] = load_x(p.x_prev, ((size_t)r * kS + sg) * H + h, p.hc_bf16);
          } else {
            // the previous layer's deferred post: X_s = sum_j comb_sj Xprev_j + post_s y
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < kS; ++j)
              acc = fmaf(pcomb[(r * kS + sg) * kS + j], load_x(p.x_prev, ((size_t)r * kS + j) * H + h, p.hc_bf16), acc);
            acc = fmaf(ppost[r * kS + sg], load_x(p.pend_y, (size_t)r * H + h, p.pend_y_bf16), acc);
            v[u] = p.hc_bf16 ? round_bf16(acc) : acc;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kXU; ++u) {
        const int i = i0 + u * kPreThreads;
        if (i < nx) {
          const int r = i / (kS * nh), sg = (i / nh) % kS, h = h0 + i % nh;
          if (!p.first) store_x(p.xbuf, ((size_t)r * kS + sg) * H + h, v[u], p.hc_bf16);
          xs[i] = v[u];
          if (p.taps.x) p.taps.x[((size_t)r * kS + sg) * H + h] = v[u];
        }
      }
    }
    cp_async_wait_all();
    bar_sync(kBarPre, kPreThreads);
    trace(p, 28, ptid == 0);
    // outputs o = r * 25 + col (col 24: the square sum), each split in P parts
    const int P = max(1, kPreThreads / nout);
    const int T = kS * nh;
    for (int op = ptid; op < nout * P; op += kPreThreads) {
      const int o = op / P, part = op % P, r = o / kMixP, col = o % kMixP;
      float acc = 0.f;
      for (int t = part; t < T; t += P) {
        const float x = xs[r * T + t];
        acc = col < kMixC ? fmaf(x, ws[t * kMixC + col], acc) : fmaf(x, x, acc);
      }
      c->red[op] = acc;
    }
    bar_sync(kBarPre, kPreThreads);
    trace(p, 17, ptid == 0);
    // partials stored output-major: mix_part[o][G]
    for (int o = ptid; o < nout; o += kPreThreads) {
      float acc = 0.f;
      for (int part = 0; part < P; ++part) acc += c->red[o * P + part];
      p.mix_part[(size_t)o * G + blockIdx.x] = acc;
    }
    if (blockIdx.x == 0)
      for (int i = ptid; i < p.n_xready_all; i += kPreThreads) p.xready[i] = 0u;
    bar_sync(kBarPre, kPreThreads);
    if (ptid == 0 && may_publish(p, c->epoch, 1, 0)) {
      red_release_add(&p.sync->cnt_mix, 1u);
    }
    trace(p, 1, ptid == 0);
  }

  if (ptid == 0) wait_count(p, c, &p.sync->cnt_mix, ep1, 1u);
  bar_sync(kBarPre, kPreThreads);
  trace(p, 2, ptid == 0);
  if (R <= 3) {
    // few outputs: every CTA's partials into shared memory at once (behind
    // the slices, which the collapse still needs), then lane-strided sums
    // and a butterfly across the warp, in the same order in every CTA.
    // The second-level counter still takes this CTA's arrival (nobody waits
    // for it in this step): its wait target counts every step, so a later
    // step with more rows finds it in step with the others.
    if (ptid == 0) red_release_add(&p.sync->cnt_mix2, 1u);
    float* parts = reinterpret_cast<float*>(regA + L.parts);
    const int cap = (int)((uint32_t)(p.regA_bytes - (int)L.parts) / 4u / (uint32_t)G);   // outputs per pass
    for (int o0 = 0; o0 < nout; o0 += cap) {
      const int no = min(cap, nout - o0);
      const int n4 = no * G / 4;   // G * 4 bytes is a multiple of 16 (the plan keeps G % 4 == 0)
      const float4* src = reinterpret_cast<const float4*>(p.mix_part + (size_t)o0 * G);
      if (!c->dead)
        for (int i = ptid; i < n4; i += kPreThreads) cp_async16(reinterpret_cast<float4*>(parts) + i, src + i);
      cp_async_commit();
      cp_async_wait_all();
      bar_sync(kBarPre, kPreThreads);
      for (int o = pwarp; o < no; o += kPreThreads / 32) {
        float acc = 0.f;
        for (int m = lane; m < G; m += 32) acc += parts[o * G + m];
        acc = warp_sum(acc);
        if (lane == 0) c->smix[(o0 + o) / kMixP][(o0 + o) % kMixP] = acc;
      }
      bar_sync(kBarPre, kPreThreads);
    }
  } else {
    // more outputs: the totals in two levels.  CTA c sums its share of the
    // outputs over every CTA's partial (the same lane-strided sums and
    // butterfly, so the same totals), publishes them, and after one more
    // grid stage every CTA reads all of them (a few hundred bytes instead of
    // every partial)
    const int o0 = (int)(blockIdx.x * (uint32_t)nout / G), o1 = (int)((blockIdx.x + 1) * (uint32_t)nout / G);
    for (int o = o0 + pwarp; o < o1; o += kPreThreads / 32) {
      float acc = 0.f;
      if (!c->dead)
        for (int m = lane; m < G; m += 32) acc += __ldcg(p.mix_part + (size_t)o * G + m);
      acc = warp_sum(acc);
      if (lane == 0) p.mix_tot[o] = acc;
    }
    bar_sync(kBarPre, kPreThreads);
    if (ptid == 0 && may_publish(p, c->epoch, 0, 10)) {
      red_release_add(&p.sync->cnt_mix2, 1u);
    }
    if (ptid == 0) wait_count(p, c, &p.sync->cnt_mix2, ep1, 1u);
    bar_sync(kBarPre, kPreThreads);
    for (int o = ptid; o < nout; o += kPreThreads) c->smix[o / kMixP][o % kMixP] = c->dead ? 0.f : __ldcg(p.mix_tot + o);
    bar_sync(kBarPre, kPreThreads);
  }
  {
    if (ptid < R) {
      const int r = ptid;
      const float rho = 1.0f / sqrtf(c->smix[r][kMixC] / (float)(kS * H) + p.rms_eps);
      for (int col = 0; col < kMixC; ++col) c->smix[r][col] *= rho;
      for (int sg = 0; sg < kS; ++sg) {
        c->pre[r][sg] = sigmoidf_(c->smix[r][sg]) + p.pre_eps;
        c->post[r][sg] = p.post_mult * sigmoidf_(c->smix[r][kS + sg]);
      }
    }
    bar_sync(kBarPre, kPreThreads);
    trace(p, 23, ptid == 0);
    if (blockIdx.x == 0) {
      for (int i = ptid; i < R * kMixC; i += kPreThreads)
        if (p.taps.mix) p.taps.mix[i] = c->smix[i / kMixC][i % kMixC];
      for (int i = ptid; i < R * kS; i += kPreThreads) {
        if (p.taps.pre) p.taps.pre[i] = c->pre[i / kS][i % kS];
        if (p.taps.post) p.taps.post[i] = c->post[i / kS][i % kS];
        if (!p.last) p.pend_out[i] = c->post[i / kS][i % kS];
      }
    }
  }
}

template <bool CANON>
__device__ __noinline__ void router_logits(const Params& p, Ctl* c, const uint8_t* n_s, bool dry);

// Control warps: Sinkhorn of the comb logits (16 threads per row), then the
// canonical top-k of each row once every CTA's router logits are out (here
// when ctl_topk; otherwise the compute warps do it in route_rows and hand
// over at the routing barrier), then the list of unique routed experts with
// their rows and act slots.
__device__ void control_warps(const Params& p, Ctl* c, const uint8_t* regA, uint32_t ep1, bool ctl_topk,
                              bool split = false) {
  const int R = p.R, E = p.E, K = p.K, G = p.G;
  const int lane = threadIdx.x & 31, cw = (threadIdx.x >> 5) - kCtlWarp0;
  const int ct = threadIdx.x - kCtlWarp0 * 32;
  for (int r0 = 0; r0 < kMaxR; r0 += kCtlWarps * 2) {
    const int r = r0 + (ct >> 4), e = ct & 15;
    const bool act = r < R;
    float lg = act ? c->smix[r][2 * kS + e] : 0.f;
    float mx = lg;
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o, 16));
    float v = expf(lg - mx);
    for (int it = 0; it < p.sink_iters; ++it) {
      float rs = v + __shfl_xor_sync(0xffffffffu, v, 1, 16);
      rs += __shfl_xor_sync(0xffffffffu, rs, 2, 16);
      v = v / rs;
      float cs = v + __shfl_xor_sync(0xffffffffu, v, 4, 16);
      cs += __shfl_xor_sync(0xffffffffu, cs, 8, 16);
      v = v / cs;
    }
    if (act) {
      c->comb[r][e] = v;
      if (blockIdx.x == 0) {
        if (p.taps.comb) p.taps.comb[r * 16 + e] = v;
        if (!p.last) p.pend_out[R * kS + r * 16 + e] = v;
      }
    }
  }
  if (ctl_topk) {
    // the top-k rows here, two warps over the rows
    if (ct == 0 && !p.dense) wait_count(p, c, &p.sync->cnt_logit, ep1, 2u);
    trace(p, 21, ct == 0);
    bar_sync(kBarCtl, kCtlWarps * 32);
    for (int r = cw; r < R; r += kCtlWarps) {
      if (p.dense) dense_row(p, c, r);
      else topk_dispatch(p, c, r, false);
    }
    for (int i = ct; i < kMaxE / 32; i += kCtlWarps * 32) c->bm[i] = 0u;
    bar_sync(kBarCtl, kCtlWarps * 32);
    trace(p, 22, ct == 0);
  } else {
    for (int i = ct; i < kMaxE / 32; i += kCtlWarps * 32) c->bm[i] = 0u;
    // idle until the compute warps have the top-k rows: run the router and
    // top-k code once without storing anything, so that it is warm in this
    // SM's instruction cache when the compute warps get there (the tensor-
    // core kernel is the only caller of this branch)
    router_logits<true>(p, c, regA, true);
    if (cw == 0) topk_dispatch(p, c, 0, true);
    // the compute warps' top-k rows (route_rows) are in c->idx / c->wt after
    // this (split: warps 4-7 alone took them)
    bar_sync(kBarRoute, split ? (4 + kCtlWarps) * 32 : kPreThreads);
  }
  for (int i = ct; i < R * K; i += kCtlWarps * 32) {
    const int e = c->idx[i / K][i % K];
    if (e >= 0 && e < E && ((c->live >> (i / K)) & 1u)) atomicOr(&c->bm[e >> 5], 1u << (e & 31));
  }
  bar_sync(kBarCtl, kCtlWarps * 32);
  if (cw == 0) {
    static_assert(kMaxE / 32 == 32, "one bitmap word per lane");
    uint32_t word = c->dead ? 0u : c->bm[lane];
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    int pos = incl - cnt;
    while (word) {
      const int b = __ffs(word) - 1;
      word &= word - 1u;
      c->ulist[pos++] = lane * 32 + b;
    }
    if (lane == 31) c->nu_ctl = incl;
  }
  bar_sync(kBarCtl, kCtlWarps * 32);
  const int nu = c->nu_ctl;
  for (int u = ct; u < nu; u += kCtlWarps * 32) {
    const int e = c->ulist[u];
    uint32_t mask = 0u;
    for (int r = 0; r < kMaxR; ++r) {
      signed char sl = -1;
      if (r < R && ((c->live >> r) & 1u))
        for (int j = 0; j < K; ++j)
          if (c->idx[r][j] == e) sl = (signed char)j;
      c->uslot[u][r] = sl;
      if (sl >= 0) mask |= 1u << r;
    }
    c->umask[u] = mask;
  }
  bar_sync(kBarCtl, kCtlWarps * 32);
  if (ct == 0) {
    c->nu = nu;
    __threadfence_block();
    *(volatile int*)&c->lists_ready = 1;
    trace(p, 5);
  }
}

// Where n (the normed rows) lives in shared memory: row-major [R][H] (bf16 if
// rounded, else fp32) for the CUDA-core kernel, or the tensor-core B operand
// layout [H/8][8 rows][8] bf16 with rows >= R zero.
template <bool CANON>
__device__ __forceinline__ size_t n_off(int r, int h, int H, bool bf) {
  if (CANON) return ((size_t)(h >> 3) * 8 + r) * 16 + (size_t)(h & 7) * 2;
  return ((size_t)r * H + h) * (bf ? 2 : 4);
}

// Collapse a = sum_s pre_s X_s (-> bf16), weighted RMSNorm n = a / sqrt(mean
// a^2 + eps) * norm_w (-> bf16), into shared memory; compute warps only.
// Each CTA collapses its own h-slice from the residual streams it staged for
// the mix, publishes it with its partial sum of a^2, and after a grid stage
// copies every slice in (one round trip) and normalises in place.
template <bool CANON>
__device__ void collapse_norm(const Params& p, Ctl* c, uint8_t* regA, uint32_t ep1) {
  const int R = p.R, H = p.H, G = p.G, ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
  const bool nbf = CANON || p.round_bf16;
  const bool abf = p.round_bf16 != 0;   // a is bf16-valued when rounded
  const PreLayout L(p);
  const int h0 = L.h0, nh = L.nh;
  {
    const float* xs = reinterpret_cast<const float*>(regA + L.xs);
    float sq[kMaxR];
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) sq[r] = 0.f;
    for (int i = ctid; i < R * nh; i += kCW * 32) {
      const int r = i / nh, hh = i % nh;
      float acc = 0.f;
#pragma unroll
      for (int sg = 0; sg < kS; ++sg) acc = fmaf(c->pre[r][sg], xs[(r * kS + sg) * nh + hh], acc);
      const float a = abf ? round_bf16(acc) : acc;
      store_x(p.abuf, (size_t)r * H + h0 + hh, a, abf);
#pragma unroll
      for (int r2 = 0; r2 < kMaxR; ++r2)
        if (r2 == r) sq[r2] = fmaf(a, a, sq[r2]);
    }
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) {
      const float v = warp_sum(sq[r]);
      if (lane == 0) c->sq[warp][r] = v;
    }
    bar_sync(kBarCons, kCW * 32);
    if (ctid < R) {
      float t = 0.f;
      for (int w = 0; w < kCW; ++w) t += c->sq[w][ctid];
      p.sq_part[(size_t)ctid * G + blockIdx.x] = t;
    }
    bar_sync(kBarCons, kCW * 32);
    if (ctid == 0 && may_publish(p, c->epoch, 7, 1)) {
      red_release_add(&p.sync->cnt_a, 1u);
    }
  }
  trace(p, 27, ctid == 0);
  if (CANON) {
    // rows R..7 of the B operand are zero (the staging areas are dead now)
    const int H8 = H / 8;
    for (int i = ctid; i < (8 - R) * H8; i += kCW * 32) {
      const int r = R + i / H8, h = (i % H8) * 8;
      *reinterpret_cast<uint4*>(regA + n_off<true>(r, h, H, true)) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (ctid == 0) wait_count(p, c, &p.sync->cnt_a, ep1, 7u);
  bar_sync(kBarCons, kCW * 32);
  trace(p, 24, ctid == 0);
  // every slice of a into the n area, 16 bytes at a time
  if (!c->dead) {
    if (abf) {
      const int H8 = H / 8;
      for (int i = ctid; i < R * H8; i += kCW * 32) {
        const int r = i / H8, h = (i % H8) * 8;
        cp_async16(regA + n_off<CANON>(r, h, H, true), reinterpret_cast<const uint16_t*>(p.abuf) + (size_t)r * H + h);
      }
    } else {   // fp32 a, row-major fp32 n (CUDA-core kernel only)
      const int H4 = H / 4;
      for (int i = ctid; i < R * H4; i += kCW * 32)
        cp_async16(regA + (size_t)i * 16, reinterpret_cast<const float*>(p.abuf) + (size_t)i * 4);
    }
  }
  cp_async_commit();
  // meanwhile: every CTA's a^2 partials, summed in the same order everywhere
  if (warp < R) {
    float t = 0.f;
    for (int m = lane; m < G; m += 32) t += c->dead ? 0.f : __ldcg(p.sq_part + (size_t)warp * G + m);
    t = warp_sum(t);
    if (lane == 0) c->inv[warp] = 1.0f / sqrtf(t / (float)H + p.rms_eps);
  }
  cp_async_wait_all();
  bar_sync(kBarCons, kCW * 32);
  trace(p, 29, ctid == 0);
  // n = a * inv * norm_w, in place: one norm_w load per 8 columns, all rows
  {
    const int H8 = H / 8;
    constexpr int kNU = 4;
    for (int i0 = ctid; i0 < H8; i0 += kNU * kCW * 32) {
      float w[kNU][8];
#pragma unroll
      for (int u = 0; u < kNU; ++u) {
        const int i = i0 + u * kCW * 32;
        if (i < H8) load_hc8(p.norm_w, (size_t)i * 8, p.norm_bf16, w[u]);
      }
#pragma unroll
      for (int u = 0; u < kNU; ++u) {
        const int i = i0 + u * kCW * 32;
        if (i >= H8) continue;
        const int h = i * 8;
        for (int r = 0; r < R; ++r) {
          float a[8];
          if (CANON) load8(regA + n_off<true>(r, h, H, true), 0, true, a);
          else load8(regA, (size_t)r * H + h, nbf, a);
          const float inv = c->inv[r];
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float v = a[k] * inv * w[u][k];
            a[k] = p.round_bf16 ? round_bf16(v) : v;
          }
          if (CANON) store8(regA + n_off<true>(r, h, H, true), 0, true, a);
          else store8(regA, (size_t)r * H + h, nbf, a);
          if (blockIdx.x == 0 && p.taps.n) {
#pragma unroll
            for (int k = 0; k < 8; ++k) p.taps.n[(size_t)r * H + h + k] = a[k];
          }
        }
      }
    }
  }
  bar_sync(kBarCons, kCW * 32);
  trace(p, 30, ctid == 0);
}

// Router logits of this CTA's experts (two rows of router_t at a time; each
// thread's share of both rows is loaded at once), then the CTA's arrival at
// the logits counter; compute warps only.  dry: the same code without
// barriers or stores, to warm the instruction cache (not inlined, so that
// both calls share the code).
template <bool CANON>
__device__ __noinline__ void router_logits(const Params& p, Ctl* c, const uint8_t* n_s, bool dry) {
  if (p.dense) return;   // no router (and no logits stage) in a dense layer
  const int R = p.R, H = p.H, E = p.E, G = p.G, ctid = threadIdx.x, warp = ctid >> 5, lane = ctid & 31;
  const bool nbf = CANON || p.round_bf16;
  const int e0 = (int)(blockIdx.x * (uint32_t)E / G), e1 = (int)((blockIdx.x + 1) * (uint32_t)E / G);
  constexpr int kRq = 5;                  // float4 per thread and row per pass
  constexpr int kSpan = kRq * kCW * 32 * 4;   // columns per pass (5120)
  for (int e = e0; e < e1; e += 2) {
    const bool two = e + 1 < e1;
    const float* w0 = p.router_t + (size_t)e * H;
    const float* w1 = two ? w0 + H : w0;
    for (int hb = 0; hb < H; hb += kSpan) {
      float4 v0[kRq], v1[kRq];
#pragma unroll
      for (int q = 0; q < kRq; ++q) {
        const int h = hb + (ctid + q * kCW * 32) * 4;
        v0[q] = h < H ? __ldg(reinterpret_cast<const float4*>(w0 + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
        v1[q] = h < H ? __ldg(reinterpret_cast<const float4*>(w1 + h)) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      // one row at a time (a rolled loop keeps this code small)
      for (int r = 0; r < R; ++r) {
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int q = 0; q < kRq; ++q) {
          const int h = hb + (ctid + q * kCW * 32) * 4;
          if (h < H) {
            float nv[4];
            if (nbf) load_vec<4, true>(n_s + n_off<CANON>(r, h, H, true), 0, nv);
            else load_vec<4, false>(n_s + n_off<CANON>(r, h, H, false), 0, nv);
            a0 = fmaf(v0[q].x, nv[0], fmaf(v0[q].y, nv[1], fmaf(v0[q].z, nv[2], fmaf(v0[q].w, nv[3], a0))));
            a1 = fmaf(v1[q].x, nv[0], fmaf(v1[q].y, nv[1], fmaf(v1[q].z, nv[2], fmaf(v1[q].w, nv[3], a1))));
          }
        }
        a0 = warp_sum(a0);
        a1 = warp_sum(a1);
        if (lane == 0 && !dry) {
          c->sq[warp][r] = (hb == 0 ? 0.f : c->sq[warp][r]) + a0;
          c->sq2[warp][r] = (hb == 0 ? 0.f : c->sq2[warp][r]) + a1;
        }
      }
    }
    if (dry) continue;
    trace(p, 25, ctid == 0 && e == e0);
    bar_sync(kBarCons, kCW * 32);
    if (ctid < 2 * R) {
      const int r = ctid % R, which = ctid / R;
      if (which == 0 || two) {
        float t = 0.f;
        for (int w = 0; w < kCW; ++w) t += which ? c->sq2[w][r] : c->sq[w][r];
        p.logits[(size_t)r * E + e + which] = t;
      }
    }
    bar_sync(kBarCons, kCW * 32);
  }
  if (dry) return;
  if (ctid == 0 && may_publish(p, c->epoch, 2, 2)) {
    red_release_add(&p.sync->cnt_logit, 1u);
  }
  trace(p, 4, ctid == 0);
}

// A6, one row per warp: wait for every CTA's logits, then the canonical
// top-k and weights of each row; the control warps take over (expert lists)
// at the routing barrier.  On all compute warps, or (split, R <= 4) on warps
// 4-7 alone while warps 0-3 go on with the shared expert.
__device__ void route_rows(const Params& p, Ctl* c, uint32_t ep1, bool split) {
  const int R = p.R, warp = threadIdx.x >> 5;
  const int w0 = split ? 4 : 0, nw = kCW - w0;
  const bool lead = (int)threadIdx.x == w0 * 32;
  if (lead && !p.dense) wait_count(p, c, &p.sync->cnt_logit, ep1, 2u);
  if (split) bar_sync(kBarTop, 4 * 32);
  else bar_sync(kBarCons, kCW * 32);
  trace(p, 21, lead);
  for (int r = warp - w0; r < R; r += nw) {
    if (p.dense) dense_row(p, c, r);
    else topk_dispatch(p, c, r, false);
  }
  trace(p, 22, lead);
  bar_sync(kBarRoute, (nw + kCtlWarps) * 32);
}

// Tail on the CTA's h-range: y = bf16(routed + shared) from yfun(r, h), then
// out_i = sum_j comb_ij X_j + post_i y (last layer) or the pending state for
// the next layer's opening expand; compute warps only.
template <class YF>
__device__ void tail(const Params& p, Ctl* c, YF yfun) {
  const int R = p.R, H = p.H, ctid = threadIdx.x;
  int h0, h1;
  Walk::dn_range(p, h0, h1);
  const int nh = h1 - h0;
  const void* X = p.first ? p.x_prev : (const void*)p.xbuf;
  float* pend_y = p.pend_out + R * kS + R * kS * kS;
  for (int i = ctid; i < R * nh; i += kCW * 32) {
    const int r = i / nh, h = h0 + i % nh;
    if (!((c->live >> r) & 1u)) continue;   // padding row: its output is left as it is
    // all loads (the residual streams and the expert outputs) before any store
    float xv[kS];
#pragma unroll
    for (int j = 0; j < kS; ++j) xv[j] = p.last ? load_x_cg(X, ((size_t)r * kS + j) * H + h, p.hc_bf16) : 0.f;
    float y = c->dead ? 0.f : yfun(r, h);
    if (p.round_bf16) y = round_bf16(y);
    if (p.taps.y) p.taps.y[(size_t)r * H + h] = y;
    if (!p.last) {
      pend_y[(size_t)r * H + h] = y;
    } else {
#pragma unroll
      for (int si = 0; si < kS; ++si) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kS; ++j) acc = fmaf(c->comb[r][si * kS + j], xv[j], acc);
        acc = fmaf(c->post[r][si], y, acc);
        store_x(p.hc_out, ((size_t)r * kS + si) * H + h, acc, p.hc_bf16);
      }
    }
  }
}

// The CTA's arrival at the end counter, with no round trip: the next launch
// on this layer slot reads the counter as the value every grid counter holds
// at its start (each takes one arrival per CTA per launch), and its CTA 0
// clears the per-expert readiness counts in its prologue.  Compute thread 0.
__device__ __forceinline__ void finish_step(const Params& p, Ctl* c, uint32_t ep1) {
  (void)ep1;
  if (threadIdx.x == 0 && !c->dead) {
    may_publish(p, c->epoch, 0, 3);
    red_release_add(&p.sync->cnt_done, 1u);
  }
}

}  // namespace mono
