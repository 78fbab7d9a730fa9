// The persistent "mono" kernel: one launch runs the whole FFN half-layer.
//
// Roles inside a CTA (384 threads):
//   warps 0-7   compute warps: mix partials, collapse + norm, router logits,
//               then every expert matvec from the weight ring, then the tail
//   warp  8     producer: issues 1-D TMA bulk copies of packed weight chunks
//               into the shared-memory ring (mbarrier complete_tx), in the
//               exact order the compute warps consume them
//   warps 9-11  control: Sinkhorn, the canonical top-k, the expert work lists
//
// Grid-wide dependencies are epoch-tagged counters in global memory (no reset
// between steps): a CTA publishes with a release-add and waits with acquire
// loads until the counter reaches (epoch + 1) * contributors.  Every wait is
// bounded by the plan's timeout; on expiry the CTA records an error word,
// raises the abort flag and runs the rest of its control flow without waiting
// (so every named barrier is still reached), then returns.
#pragma once
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
constexpr int kCW = 8;        // compute warps == items per ring stage
constexpr int kProdWarp = 8;
constexpr int kCtlWarp0 = 9;
constexpr int kCtlWarps = 3;
constexpr int kThreads = (kCW + 1 + kCtlWarps) * 32;   // 384: 12 warps leave 168 registers a thread
constexpr int kPreThreads = (kCW + kCtlWarps) * 32;    // compute + control
constexpr int kBarPre = 1, kBarCons = 2, kBarCtl = 3;

enum WType { W_F32 = 0, W_BF16 = 1, W_FP8 = 2, W_FP4 = 3 };

struct SyncBlock {   // one per layer slot, 64 bytes
  uint32_t epoch, cnt_mix, cnt_logit, cnt_act, cnt_done, pad[11];
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
  int mix_ctas;
  int hc_bf16, norm_bf16, round_bf16;
  float rms_eps, pre_eps, post_mult, route_scale, denom_clamp;
  int sink_iters;
  // residual streams
  const void* x_prev;   // first: this layer's X (hc_in); else the previous layer's X
  void* xbuf;           // this layer's X when not first (written by the mix CTAs)
  void* hc_out;         // written when last
  const float* pend_in; // previous layer's pending post [R][4] | comb [R][16] | y [R][H]
  float* pend_out;      // this layer's pending state (when not last)
  // packed weights
  const float* mix_w;
  const void* norm_w;
  const float* router_t;   // [E][H]
  const float* bias;
  const uint8_t* gu;       // [E+1][I][gu_nk][2][gu_rc]
  const uint8_t* dn;       // [E+1][H][dn_nk][dn_rc]
  int gu_kc, gu_nk, gu_rc;
  int dn_kc, dn_nk, dn_rc;
  long long gu_estride, dn_estride;
  // scratch
  float* mix_part;   // [R*25][G] output-major partials of the mix
  float* logits;     // [R][E]
  float* act;        // [R][K+1][I]
  SyncBlock* sync;
  ErrBlock* err;
  Taps taps;
  int nst, slot_bytes, regA_bytes, ymax;
  unsigned long long timeout_ns;
  int fault_cta;
  unsigned long long* trace;   // optional [G][kTracePoints] globaltimer stamps
};

constexpr int kTracePoints = 16;
// stage timestamps (one writer per point and CTA)
__device__ __forceinline__ void trace(const Params& p, int point, bool who = true) {
  if (p.trace && who) p.trace[blockIdx.x * kTracePoints + point] = globaltimer();
}

// per-CTA control block in shared memory
struct Ctl {
  volatile int dead;
  volatile int lists_ready;
  uint32_t epoch;
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
    total = ring + (size_t)nst * slot_bytes;
  }
};

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
  uint32_t ns = 32;
  while (true) {
    if (*dead) return false;
    uint32_t v = ld_acquire(cnt);
    if ((int32_t)(v - target) >= 0) return true;
    if (ld_relaxed(&p.err->abort)) {
      c->dead = 1;
      return false;
    }
    if (globaltimer() - t0 > p.timeout_ns) {
      record_error(p, c, 7u, stage);   // MONO_ERR_DEVICE_TIMEOUT (negated on the host)
      return false;
    }
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
  }
}

__device__ bool wait_bar(const Params& p, Ctl* c, uint64_t* bar, uint32_t parity) {
  volatile int* dead = &c->dead;
  if (mbar_test(bar, parity)) return true;
  uint64_t t0 = globaltimer();
  while (true) {
    if (*dead) return false;
    if (mbar_test(bar, parity)) return true;
    if (globaltimer() - t0 > 2 * p.timeout_ns) {   // downstream of the grid-wide waits
      record_error(p, c, 7u, 5u);
      return false;
    }
    __nanosleep(20);
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

// ------------------------------------------------------------- expert math --
// A weight unit is 16 bytes of codes.  Products are formed on fp32 pairs with
// the packed FFMA2 instruction (fma.rn.f32x2): an accumulator pair holds the
// sums over the even and over the odd contraction positions.

__device__ __forceinline__ void ffma2(float2& d, float2 a, float2 b) {
  asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n mov.b64 rd, {%0, %1};\n"
      " fma.rn.f32x2 rd, ra, rb, rd;\n mov.b64 {%0, %1}, rd;\n}\n"
      : "+f"(d.x), "+f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
}

__device__ __forceinline__ float2 bf16x2_f2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }

// weights decoded per sub-block of SUB elements (SUB / 2 pairs)
template <int WT> struct Sub { static constexpr int N = 8; };
template <> struct Sub<W_F32> { static constexpr int N = 4; };

template <int WT> __device__ __forceinline__ void decode_sub(const uint4& q, int b, float2* w);
template <> __device__ __forceinline__ void decode_sub<W_F32>(const uint4& q, int, float2* w) {
  w[0] = make_float2(__uint_as_float(q.x), __uint_as_float(q.y));
  w[1] = make_float2(__uint_as_float(q.z), __uint_as_float(q.w));
}
template <> __device__ __forceinline__ void decode_sub<W_BF16>(const uint4& q, int, float2* w) {
  w[0] = bf16x2_f2(q.x);
  w[1] = bf16x2_f2(q.y);
  w[2] = bf16x2_f2(q.z);
  w[3] = bf16x2_f2(q.w);
}
template <> __device__ __forceinline__ void decode_sub<W_FP8>(const uint4& q, int b, float2* w) {
  const uint32_t a = b == 0 ? q.x : q.z, c = b == 0 ? q.y : q.w;
  w[0] = e4m3x2_to_f2((uint16_t)(a & 0xFFFFu));
  w[1] = e4m3x2_to_f2((uint16_t)(a >> 16));
  w[2] = e4m3x2_to_f2((uint16_t)(c & 0xFFFFu));
  w[3] = e4m3x2_to_f2((uint16_t)(c >> 16));
}
template <> __device__ __forceinline__ void decode_sub<W_FP4>(const uint4& q, int b, float2* w) {
  const uint32_t a = b == 0 ? q.x : b == 1 ? q.y : b == 2 ? q.z : q.w;
  w[0] = e2m1x2_to_f2(a & 0xFFu);
  w[1] = e2m1x2_to_f2((a >> 8) & 0xFFu);
  w[2] = e2m1x2_to_f2((a >> 16) & 0xFFu);
  w[3] = e2m1x2_to_f2(a >> 24);
}

// SUB activation values starting at element k of a row, as pairs
template <int SUB, bool BF>
__device__ __forceinline__ void load_pairs(const uint8_t* row, int k, float2* a) {
  if (BF) {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(row) + k;
    if (SUB % 8 == 0) {
#pragma unroll
      for (int i = 0; i < SUB / 8; ++i) {
        const uint4 v = reinterpret_cast<const uint4*>(src)[i];
        a[4 * i] = bf16x2_f2(v.x);
        a[4 * i + 1] = bf16x2_f2(v.y);
        a[4 * i + 2] = bf16x2_f2(v.z);
        a[4 * i + 3] = bf16x2_f2(v.w);
      }
    } else {
      const uint2 v = *reinterpret_cast<const uint2*>(src);
      a[0] = bf16x2_f2(v.x);
      a[1] = bf16x2_f2(v.y);
    }
  } else {
    const float* src = reinterpret_cast<const float*>(row) + k;
#pragma unroll
    for (int i = 0; i < SUB / 4; ++i) {
      const float4 v = reinterpret_cast<const float4*>(src)[i];
      a[2 * i] = make_float2(v.x, v.y);
      a[2 * i + 1] = make_float2(v.z, v.w);
    }
  }
}

template <int M> struct RowPtrs {
  const uint8_t* p[M];
};

// One gate/up row-chunk pair ([gate codes | scales][up codes | scales], rc
// bytes each) against the M active rows of n.
template <int WT, bool NBF, int M>
__device__ __forceinline__ void gu_chunk(const uint8_t* gch, int rc, int kc, int k0, const RowPtrs<M>& nr,
                                         float2 (&ag)[M], float2 (&au)[M]) {
  constexpr int EPU = WFmt<WT>::EPU, SUB = Sub<WT>::N, NSB = EPU / SUB;
  constexpr bool SC = (WT == W_FP8 || WT == W_FP4);
  const int lane = threadIdx.x & 31;
  const int nunits = units_of<WT>(kc);
  const uint8_t* uch = gch + rc;
#pragma unroll 2
  for (int u = lane; u < nunits; u += 32) {
    const uint4 gq = reinterpret_cast<const uint4*>(gch)[u];
    const uint4 uq = reinterpret_cast<const uint4*>(uch)[u];
    const int kb = k0 + u * EPU;
    float2 pg[M], pu[M];
#pragma unroll
    for (int t = 0; t < M; ++t) {
      pg[t] = make_float2(0.f, 0.f);
      pu[t] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int b = 0; b < NSB; ++b) {
      float2 gw[SUB / 2], uw[SUB / 2];
      decode_sub<WT>(gq, b, gw);
      decode_sub<WT>(uq, b, uw);
#pragma unroll
      for (int t = 0; t < M; ++t) {
        float2 nv[SUB / 2];
        load_pairs<SUB, NBF>(nr.p[t], kb + b * SUB, nv);
#pragma unroll
        for (int i = 0; i < SUB / 2; ++i) {
          ffma2(SC ? pg[t] : ag[t], gw[i], nv[i]);
          ffma2(SC ? pu[t] : au[t], uw[i], nv[i]);
        }
      }
    }
    if (SC) {
      const float sg = unit_scale<WT>(gch, kc, u), su = unit_scale<WT>(uch, kc, u);
#pragma unroll
      for (int t = 0; t < M; ++t) {
        ffma2(ag[t], pg[t], make_float2(sg, sg));
        ffma2(au[t], pu[t], make_float2(su, su));
      }
    }
  }
}

// One down row-chunk against the M active rows of act (fp32 [M][I] in smem).
template <int WT, int M>
__device__ __forceinline__ void dn_chunk(const uint8_t* ch, int kc, int k0, const RowPtrs<M>& ar, float2 (&ad)[M]) {
  constexpr int EPU = WFmt<WT>::EPU, SUB = Sub<WT>::N, NSB = EPU / SUB;
  constexpr bool SC = (WT == W_FP8 || WT == W_FP4);
  const int lane = threadIdx.x & 31;
  const int nunits = units_of<WT>(kc);
#pragma unroll 2
  for (int u = lane; u < nunits; u += 32) {
    const uint4 wq = reinterpret_cast<const uint4*>(ch)[u];
    const int kb = k0 + u * EPU;
    float2 pd[M];
#pragma unroll
    for (int t = 0; t < M; ++t) pd[t] = make_float2(0.f, 0.f);
#pragma unroll
    for (int b = 0; b < NSB; ++b) {
      float2 ww[SUB / 2];
      decode_sub<WT>(wq, b, ww);
#pragma unroll
      for (int t = 0; t < M; ++t) {
        float2 av[SUB / 2];
        load_pairs<SUB, false>(ar.p[t], kb + b * SUB, av);
#pragma unroll
        for (int i = 0; i < SUB / 2; ++i) ffma2(SC ? pd[t] : ad[t], ww[i], av[i]);
      }
    }
    if (SC) {
      const float sc = unit_scale<WT>(ch, kc, u);
#pragma unroll
      for (int t = 0; t < M; ++t) ffma2(ad[t], pd[t], make_float2(sc, sc));
    }
  }
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

// Router select of one row by one warp: score = sqrt(softplus(logit)) in
// fp32, sel = score + bias, canonical top-k by (sel desc, index asc) through
// warp max / min reductions, then weight = score / max(sum, clamp) * scale
// with each op rounded to fp32.  Lane l holds experts l + 32 q, q < NQ.
template <int NQ>
__device__ __forceinline__ void topk_row(const Params& p, Ctl* c, int r) {
  const int lane = threadIdx.x & 31;
  const int E = p.E, K = p.K;
  float score[NQ];
  uint32_t key[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int e = lane + 32 * q;
    score[q] = 0.f;
    key[q] = 0u;
    if (e < E) {
      const float lg = c->dead ? 0.f : __ldcg(p.logits + (size_t)r * E + e);
      if (blockIdx.x == 0 && p.taps.logits) p.taps.logits[(size_t)r * E + e] = lg;
      const float sp = fmaxf(lg, 0.f) + log1pf(expf(-fabsf(lg)));
      score[q] = sqrtf(sp);
      key[q] = ord_key(score[q] + __ldg(p.bias + e));
    }
  }
  uint32_t taken = 0u;
  float ssum = 0.f;
  for (int j = 0; j < K; ++j) {
    uint32_t bk = 0u;
    int be = 0x7FFFFFFF;
    float bs = 0.f;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      if (!((taken >> q) & 1u) && key[q] > bk) {
        bk = key[q];
        be = lane + 32 * q;
        bs = score[q];
      }
    }
    const uint32_t wk = __reduce_max_sync(0xffffffffu, bk);
    const int we = (int)__reduce_min_sync(0xffffffffu, (uint32_t)(bk == wk ? be : 0x7FFFFFFF));
    const int wl = we & 31;
    if (we < E && wl == lane) taken |= 1u << (we >> 5);
    const float ws = __shfl_sync(0xffffffffu, bs, wl);
    if (lane == 0) {
      c->idx[r][j] = we < E ? we : 0;
      c->wt[r][j] = ws;   // the raw score until the sum is known
    }
    ssum += ws;   // selection order, fp32
  }
  __syncwarp();
  if (lane < K) {
    const float den = fmaxf(ssum, p.denom_clamp);
    const float w = __fmul_rn(__fdiv_rn(c->wt[r][lane], den), p.route_scale);
    c->wt[r][lane] = w;
    if (blockIdx.x == 0) {
      if (p.taps.idx) p.taps.idx[r * K + lane] = c->idx[r][lane];
      if (p.taps.w) p.taps.w[r * K + lane] = w;
    }
  }
  __syncwarp();
}

// ------------------------------------------------------------ work walkers --

// The stage sequence of one CTA.  Producer and consumers run the same walker;
// a stage is (phase, expert slot, first item, items, chunk index).
enum Phase { PH_SGU = 0, PH_RGU = 1, PH_DN = 2 };

struct Walk {
  // shared expert gate/up: channels [c0, c1)
  __device__ static void sgu_range(const Params& p, int& c0, int& c1) {
    c0 = (int)((long long)blockIdx.x * p.I / p.G);
    c1 = (int)((long long)(blockIdx.x + 1) * p.I / p.G);
  }
  // routed gate/up over the unique-expert list: global channels [g0, g1)
  __device__ static void rgu_range(const Params& p, int nu, long long& g0, long long& g1) {
    long long n = (long long)nu * p.I;
    g0 = (long long)blockIdx.x * n / p.G;
    g1 = (long long)(blockIdx.x + 1) * n / p.G;
  }
  // down: output channels [h0, h1) of every expert
  __device__ static void dn_range(const Params& p, int& h0, int& h1) {
    h0 = (int)((long long)blockIdx.x * p.H / p.G);
    h1 = (int)((long long)(blockIdx.x + 1) * p.H / p.G);
  }
};

// --------------------------------------------------------------- the kernel --

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) mono_ffn_layer_kernel(const Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const SmemLayout L(p.nst, p.slot_bytes, p.regA_bytes, p.ymax);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + p.nst;
  Ctl* c = reinterpret_cast<Ctl*>(smem + L.ctl);
  float* ys = reinterpret_cast<float*>(smem + L.ys);
  uint8_t* regA = smem + L.regA;
  uint8_t* ring = smem + L.ring;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int R = p.R, H = p.H, I = p.I, E = p.E, K = p.K, G = p.G;
  const bool nbf = p.round_bf16 != 0;   // n is stored as bf16 exactly when it is rounded to bf16

  if (tid == 0) {
    c->dead = 0;
    c->lists_ready = 0;
    c->nu = 0;
    c->epoch = ld_relaxed(&p.sync->epoch);
    if (ld_relaxed(&p.err->abort)) c->dead = 1;   // fail-stop after an unreported error
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    fence_barrier_init();
  }
  __syncthreads();
  if (c->dead) return;
  const uint32_t ep1 = c->epoch + 1u;
  trace(p, 0, tid == 0);

  // ================================================================ producer
  if (warp == kProdWarp) {
    int h0, h1, c0, c1;
    Walk::dn_range(p, h0, h1);
    Walk::sgu_range(p, c0, c1);
    // Early L2 prefetch of everything this CTA reads before the routing is known.
    if (lane == 0) {
      auto pf = [&](const void* src, long long bytes) {
        const uint8_t* s8 = reinterpret_cast<const uint8_t*>(src);
        for (long long o = 0; o < bytes; o += 65536) {
          long long n = bytes - o < 65536 ? bytes - o : 65536;
          if ((n & ~15ll) > 0) prefetch_l2(s8 + o, (uint32_t)(n & ~15ll));
        }
      };
      int e0 = (int)((long long)blockIdx.x * E / G), e1 = (int)((long long)(blockIdx.x + 1) * E / G);
      if (e1 > e0) pf(p.router_t + (size_t)e0 * H, (long long)(e1 - e0) * H * 4);
      if (c1 > c0)
        pf(p.gu + (size_t)E * p.gu_estride + (size_t)c0 * p.gu_nk * 2 * p.gu_rc,
           (long long)(c1 - c0) * p.gu_nk * 2 * p.gu_rc);
      if (h1 > h0)
        pf(p.dn + (size_t)E * p.dn_estride + (size_t)h0 * p.dn_nk * p.dn_rc, (long long)(h1 - h0) * p.dn_nk * p.dn_rc);
    }
    __syncwarp();
    uint32_t s = 0;        // stage counter
    uint32_t issued = 0;   // stages actually issued (a prefix of the sequence)
    bool ok = true;
    auto issue = [&](const uint8_t* base, long long item_stride, int item_bytes, int n) {
      const uint32_t slot = s % p.nst, q = s / p.nst;
      if (ok && q > 0 && lane == 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      if (ok) {
        if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)(n * item_bytes));
        __syncwarp();
        if (lane < n)
          tma_load_1d(ring + (size_t)slot * p.slot_bytes + (size_t)lane * item_bytes, base + (size_t)lane * item_stride,
                      (uint32_t)item_bytes, &full[slot]);
        issued = s + 1;
      }
      ++s;
    };
    const long long gu_item = (long long)p.gu_nk * 2 * p.gu_rc;
    const long long dn_item = (long long)p.dn_nk * p.dn_rc;
    // shared gate/up
    for (int g = c0; g < c1; g += kCW) {
      int n = min(kCW, c1 - g);
      for (int k = 0; k < p.gu_nk; ++k)
        issue(p.gu + (size_t)E * p.gu_estride + (size_t)g * gu_item + (size_t)k * 2 * p.gu_rc, gu_item, 2 * p.gu_rc, n);
    }
    // routed gate/up: needs the work lists
    if (ok && lane == 0) ok = wait_flag(p, c, &c->lists_ready);
    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    const int nu = ok ? *(volatile int*)&c->nu : 0;
    trace(p, 11, lane == 0);
    // put the first part of this CTA's routed gate/up rows on their way to L2
    // while the ring still drains the shared expert
    if (lane == 0 && ok) {
      long long g0, g1;
      Walk::rgu_range(p, nu, g0, g1);
      long long budget = 256 << 10;
      const long long row = (long long)p.gu_nk * 2 * p.gu_rc;
      while (g0 < g1 && budget > 0) {
        const int u = (int)(g0 / I), ch = (int)(g0 % I);
        const long long n = min((long long)I - ch, g1 - g0);
        const long long bytes = min(n * row, budget);
        const uint8_t* src = p.gu + (size_t)c->ulist[u] * p.gu_estride + (size_t)ch * row;
        for (long long o = 0; o < bytes; o += 65536) {
          const long long b = min(65536ll, bytes - o) & ~15ll;
          if (b > 0) prefetch_l2(src + o, (uint32_t)b);
        }
        budget -= bytes;
        g0 += n;
      }
    }
    {
      long long g0, g1;
      Walk::rgu_range(p, nu, g0, g1);
      long long gch = g0;
      while (gch < g1) {
        int u = (int)(gch / I), ch = (int)(gch % I);
        int end = min((long long)I, ch + (g1 - gch));
        int e = c->ulist[u];
        for (int g = ch; g < end; g += kCW) {
          int n = min(kCW, end - g);
          for (int k = 0; k < p.gu_nk; ++k)
            issue(p.gu + (size_t)e * p.gu_estride + (size_t)g * gu_item + (size_t)k * 2 * p.gu_rc, gu_item, 2 * p.gu_rc,
                  n);
        }
        gch += end - ch;
      }
    }
    // down projections: shared first, then the routed list in order
    for (int x = 0; x <= nu; ++x) {
      int e = x == 0 ? E : c->ulist[x - 1];
      for (int g = h0; g < h1; g += kCW) {
        int n = min(kCW, h1 - g);
        for (int k = 0; k < p.dn_nk; ++k)
          issue(p.dn + (size_t)e * p.dn_estride + (size_t)g * dn_item + (size_t)k * p.dn_rc, dn_item, p.dn_rc, n);
      }
    }
    trace(p, 12, lane == 0);
    // drain: no bulk copy may still target this CTA's shared memory at exit
    if (lane == 0) {
      uint32_t first = issued > (uint32_t)p.nst ? issued - p.nst : 0;
      for (uint32_t t = first; t < issued; ++t) {
        uint32_t slot = t % p.nst, q = t / p.nst;
        uint64_t t0 = globaltimer();
        while (!mbar_test(&full[slot], q & 1)) {
          if (globaltimer() - t0 > p.timeout_ns) break;
          __nanosleep(64);
        }
      }
    }
    return;
  }

  // ============================================ A2: mix partials (+ expand)
  // compute + control warps; every CTA takes the h-range it also owns in the
  // down projections and the tail
  const int ptid = warp < kCW ? tid : tid - 32;   // 0 .. kPreThreads-1 over compute and control warps
  const int pwarp = ptid >> 5;
  const int nout = R * kMixP;
  {
    int h0, h1;
    Walk::dn_range(p, h0, h1);
    const int nh = h1 - h0;
    float* ws = reinterpret_cast<float*>(regA);          // [S][nh][24] slice of mix_w
    float* xs = ws + (size_t)kS * nh * kMixC;            // [R][S][nh]
    // the mix_w slice: S contiguous segments of nh rows x 24 fp32 (96 bytes a row)
    const int seg4 = nh * (kMixC / 4);
    for (int i = ptid; i < kS * seg4; i += kPreThreads) {
      const int sgm = i / seg4, j = i % seg4;
      reinterpret_cast<float4*>(ws)[i] =
          __ldg(reinterpret_cast<const float4*>(p.mix_w + ((size_t)sgm * H + h0) * kMixC) + j);
    }
    const float* ppost = p.pend_in;
    const float* pcomb = p.pend_in + R * kS;
    const float* py = p.pend_in + R * kS + R * kS * kS;
    for (int i = ptid; i < R * kS * nh; i += kPreThreads) {
      const int r = i / (kS * nh), sg = (i / nh) % kS, h = h0 + i % nh;
      float v;
      if (p.first) {
        v = load_x(p.x_prev, ((size_t)r * kS + sg) * H + h, p.hc_bf16);
      } else {
        // the previous layer's deferred post: X_s = sum_j comb_sj Xprev_j + post_s y
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < kS; ++j)
          acc = fmaf(pcomb[(r * kS + sg) * kS + j], load_x(p.x_prev, ((size_t)r * kS + j) * H + h, p.hc_bf16), acc);
        acc = fmaf(ppost[r * kS + sg], py[(size_t)r * H + h], acc);
        v = p.hc_bf16 ? round_bf16(acc) : acc;
        store_x(p.xbuf, ((size_t)r * kS + sg) * H + h, v, p.hc_bf16);
      }
      xs[i] = v;
      if (p.taps.x) p.taps.x[((size_t)r * kS + sg) * H + h] = v;
    }
    bar_sync(kBarPre, kPreThreads);
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
    // partials stored output-major: mix_part[o][G]
    for (int o = ptid; o < nout; o += kPreThreads) {
      float acc = 0.f;
      for (int part = 0; part < P; ++part) acc += c->red[o * P + part];
      p.mix_part[(size_t)o * G + blockIdx.x] = acc;
    }
    bar_sync(kBarPre, kPreThreads);
    if (ptid == 0) {
      __threadfence();
      red_release_add(&p.sync->cnt_mix, 1u);
    }
    trace(p, 1, ptid == 0);
  }

  // ======================================= A3: mix totals, pre, post (all)
  if (ptid == 0) wait_count(p, c, &p.sync->cnt_mix, ep1 * (uint32_t)G, 1u);
  bar_sync(kBarPre, kPreThreads);
  trace(p, 2, ptid == 0);
  {
    // every CTA reduces the G partials of every output in the same fixed order:
    // lane-strided sums, then a butterfly across the warp
    float* parts = reinterpret_cast<float*>(regA);
    const int cap = p.regA_bytes / (int)sizeof(float) / G;   // outputs per pass
    for (int o0 = 0; o0 < nout; o0 += cap) {
      const int no = min(cap, nout - o0);
      const int n4 = no * G / 4;   // G * 4 bytes is a multiple of 16 (the plan keeps G % 4 == 0)
      const float4* src = reinterpret_cast<const float4*>(p.mix_part + (size_t)o0 * G);
      for (int i = ptid; i < n4; i += kPreThreads) reinterpret_cast<float4*>(parts)[i] = c->dead ? make_float4(0.f, 0.f, 0.f, 0.f) : __ldcg(src + i);
      bar_sync(kBarPre, kPreThreads);
      for (int o = pwarp; o < no; o += kPreThreads / 32) {
        float acc = 0.f;
        for (int m = lane; m < G; m += 32) acc += parts[o * G + m];
        acc = warp_sum(acc);
        if (lane == 0) c->smix[(o0 + o) / kMixP][(o0 + o) % kMixP] = acc;
      }
      bar_sync(kBarPre, kPreThreads);
    }
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
    if (blockIdx.x == 0) {
      for (int i = ptid; i < R * kMixC; i += kPreThreads) {
        if (p.taps.mix) p.taps.mix[i] = c->smix[i / kMixC][i % kMixC];
      }
      for (int i = ptid; i < R * kS; i += kPreThreads) {
        if (p.taps.pre) p.taps.pre[i] = c->pre[i / kS][i % kS];
        if (p.taps.post) p.taps.post[i] = c->post[i / kS][i % kS];
        if (!p.last) p.pend_out[i] = c->post[i / kS][i % kS];
      }
    }
  }

  // ====================================================== control warps
  if (warp >= kCtlWarp0) {
    const int ct = tid - kCtlWarp0 * 32;   // 0 .. kCtlWarps * 32 - 1
    // Sinkhorn of exp(comb logits): 16 threads per row (one per entry), rows
    // in passes of kCtlWarps * 2
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
    // wait for every CTA's router logits
    if (ct == 0) wait_count(p, c, &p.sync->cnt_logit, ep1 * (uint32_t)G, 2u);
    bar_sync(kBarCtl, kCtlWarps * 32);
    const int cw = warp - kCtlWarp0;
    for (int r = cw; r < R; r += kCtlWarps) {
      if (E <= 32) topk_row<1>(p, c, r);
      else if (E <= 64) topk_row<2>(p, c, r);
      else if (E <= 128) topk_row<4>(p, c, r);
      else if (E <= 256) topk_row<8>(p, c, r);
      else if (E <= 512) topk_row<16>(p, c, r);
      else topk_row<32>(p, c, r);
    }
    // unique routed experts in ascending order, with their rows and act slots:
    // a bitmap of the selected experts, a warp scan of its popcounts, then one
    // thread per unique expert
    for (int i = ct; i < kMaxE / 32; i += kCtlWarps * 32) c->bm[i] = 0u;
    bar_sync(kBarCtl, kCtlWarps * 32);
    for (int i = ct; i < R * K; i += kCtlWarps * 32) {
      const int e = c->idx[i / K][i % K];
      if (e >= 0 && e < E) atomicOr(&c->bm[e >> 5], 1u << (e & 31));
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
        if (r < R)
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
    return;
  }

  // ================================================ compute warps from here
  const int ctid = tid;   // 0..255
  // ---------------- collapse + weighted RMSNorm: n [R][H] in region A
  {
    const void* X = p.first ? p.x_prev : (const void*)p.xbuf;
    const int H8 = H / 8;
    float sq[kMaxR];
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) sq[r] = 0.f;
#pragma unroll 2
    for (int i = ctid; i < R * H8; i += kCW * 32) {
      const int r = i / H8, h = (i % H8) * 8;
      float xv[kS][8];
#pragma unroll
      for (int sg = 0; sg < kS; ++sg) load_hc8(X, ((size_t)r * kS + sg) * H + h, p.hc_bf16, xv[sg]);
      float a[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        float acc = 0.f;
#pragma unroll
        for (int sg = 0; sg < kS; ++sg) acc = fmaf(c->pre[r][sg], xv[sg][k], acc);
        a[k] = p.round_bf16 ? round_bf16(acc) : acc;
      }
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < 8; ++k) q = fmaf(a[k], a[k], q);
#pragma unroll
      for (int r2 = 0; r2 < kMaxR; ++r2)
        if (r2 == r) sq[r2] += q;
      store8(regA, (size_t)r * H + h, nbf, a);
    }
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) {
      float v = warp_sum(sq[r]);
      if (lane == 0) c->sq[warp][r] = v;
    }
    bar_sync(kBarCons, kCW * 32);
    if (ctid < R) {
      float t = 0.f;
      for (int w = 0; w < kCW; ++w) t += c->sq[w][ctid];
      c->inv[ctid] = 1.0f / sqrtf(t / (float)H + p.rms_eps);
    }
    bar_sync(kBarCons, kCW * 32);
#pragma unroll 2
    for (int i = ctid; i < R * H8; i += kCW * 32) {
      const int r = i / H8, h = (i % H8) * 8;
      float a[8], w[8];
      load8(regA, (size_t)r * H + h, nbf, a);
      load_hc8(p.norm_w, h, p.norm_bf16, w);
      const float inv = c->inv[r];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float v = a[k] * inv * w[k];
        a[k] = p.round_bf16 ? round_bf16(v) : v;
      }
      store8(regA, (size_t)r * H + h, nbf, a);
      if (blockIdx.x == 0 && p.taps.n) {
#pragma unroll
        for (int k = 0; k < 8; ++k) p.taps.n[(size_t)r * H + h + k] = a[k];
      }
    }
    bar_sync(kBarCons, kCW * 32);
  }
  const void* n_s = regA;
  trace(p, 3, ctid == 0);

  // ---------------- router logits for this CTA's experts, two rows of
  // router_t at a time with every load of the pass issued up front
  {
    const int e0 = (int)((long long)blockIdx.x * E / G), e1 = (int)((long long)(blockIdx.x + 1) * E / G);
    for (int e = e0; e < e1; e += 2) {
      const bool two = e + 1 < e1;
      const float* w0 = p.router_t + (size_t)e * H;
      const float* w1 = two ? w0 + H : w0;
      float a0[kMaxR], a1[kMaxR];
#pragma unroll
      for (int r = 0; r < kMaxR; ++r) { a0[r] = 0.f; a1[r] = 0.f; }
#pragma unroll 4
      for (int h = ctid * 4; h < H; h += kCW * 32 * 4) {
        const float4 v0 = __ldg(reinterpret_cast<const float4*>(w0 + h));
        const float4 v1 = __ldg(reinterpret_cast<const float4*>(w1 + h));
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) {
          if (r < R) {
            float nv[4];
            if (nbf) load_vec<4, true>((const uint16_t*)n_s + (size_t)r * H, h, nv);
            else load_vec<4, false>((const float*)n_s + (size_t)r * H, h, nv);
            a0[r] = fmaf(v0.x, nv[0], fmaf(v0.y, nv[1], fmaf(v0.z, nv[2], fmaf(v0.w, nv[3], a0[r]))));
            a1[r] = fmaf(v1.x, nv[0], fmaf(v1.y, nv[1], fmaf(v1.z, nv[2], fmaf(v1.w, nv[3], a1[r]))));
          }
        }
      }
#pragma unroll
      for (int r = 0; r < kMaxR; ++r) {
        const float v0 = warp_sum(a0[r]);
        const float v1 = warp_sum(a1[r]);
        if (lane == 0) {
          c->sq[warp][r] = v0;
          c->sq2[warp][r] = v1;
        }
      }
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
    if (ctid == 0 && (int)blockIdx.x != p.fault_cta) {
      __threadfence();
      red_release_add(&p.sync->cnt_logit, 1u);
    }
    trace(p, 4, ctid == 0);
  }

  // ---------------- expert matvecs from the weight ring
  uint32_t s = 0;   // stage counter (mirrors the producer)
  auto stage_wait = [&](uint32_t st) -> const uint8_t* {
    const uint32_t slot = st % p.nst, q = st / p.nst;
    if (!mbar_test(&full[slot], q & 1)) wait_bar(p, c, &full[slot], q & 1);
    return ring + (size_t)slot * p.slot_bytes;
  };
  auto stage_release = [&](uint32_t st) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[st % p.nst]);
  };
  const size_t n_row_bytes = (size_t)H * (nbf ? 2 : 4);

  // gate/up of one expert: channels [g, g + n) of warp-sized groups; rows and
  // act slots of the M active rows packed 4 and 8 bits per entry
  auto gu_group = [&](auto Mc, int g, int n, uint32_t rows4, uint64_t slots8) {
    constexpr int M = decltype(Mc)::value;
    RowPtrs<M> nr;
#pragma unroll
    for (int t = 0; t < M; ++t) nr.p[t] = regA + (size_t)((rows4 >> (4 * t)) & 15u) * n_row_bytes;
    float2 ag[M], au[M];
#pragma unroll
    for (int t = 0; t < M; ++t) {
      ag[t] = make_float2(0.f, 0.f);
      au[t] = make_float2(0.f, 0.f);
    }
    const bool mine = warp < n;
    for (int k = 0; k < p.gu_nk; ++k) {
      const uint8_t* st = stage_wait(s);
      if (mine && !c->dead) {
        const uint8_t* it = st + (size_t)warp * 2 * p.gu_rc;
        if (nbf) gu_chunk<WT, true, M>(it, p.gu_rc, p.gu_kc, k * p.gu_kc, nr, ag, au);
        else gu_chunk<WT, false, M>(it, p.gu_rc, p.gu_kc, k * p.gu_kc, nr, ag, au);
      }
      stage_release(s);
      ++s;
    }
    if (mine) {
#pragma unroll
      for (int t = 0; t < M; ++t) {
        float gsum = warp_sum(ag[t].x + ag[t].y);
        float usum = warp_sum(au[t].x + au[t].y);
        if (lane == t) {
          if (p.round_bf16) {
            gsum = round_bf16(gsum);
            usum = round_bf16(usum);
          }
          const float a = gsum / (1.0f + expf(-gsum)) * usum;
          const uint32_t r = (rows4 >> (4 * t)) & 15u, sl = (uint32_t)(slots8 >> (8 * t)) & 255u;
          p.act[((size_t)r * (K + 1) + sl) * I + g + warp] = a;
        }
      }
    }
  };
  auto dispatch_gu = [&](int M, int g, int n, uint32_t rows4, uint64_t slots8) {
    switch (M) {
      case 1: gu_group(std::integral_constant<int, 1>{}, g, n, rows4, slots8); break;
      case 2: gu_group(std::integral_constant<int, 2>{}, g, n, rows4, slots8); break;
      case 3: gu_group(std::integral_constant<int, 3>{}, g, n, rows4, slots8); break;
      case 4: gu_group(std::integral_constant<int, 4>{}, g, n, rows4, slots8); break;
      case 5: gu_group(std::integral_constant<int, 5>{}, g, n, rows4, slots8); break;
      case 6: gu_group(std::integral_constant<int, 6>{}, g, n, rows4, slots8); break;
      case 7: gu_group(std::integral_constant<int, 7>{}, g, n, rows4, slots8); break;
      default: gu_group(std::integral_constant<int, 8>{}, g, n, rows4, slots8); break;
    }
  };
  // rows / act slots of unique-expert entry x (x == 0: the shared expert)
  auto expert_rows = [&](int x, uint32_t& rows4, uint64_t& slots8) -> int {
    int M = 0;
    rows4 = 0u;
    slots8 = 0ull;
    for (int r = 0; r < R; ++r) {
      int sl = -1;
      if (x == 0) sl = K;
      else if ((c->umask[x - 1] >> r) & 1u) sl = c->uslot[x - 1][r];
      if (sl >= 0) {
        rows4 |= (uint32_t)r << (4 * M);
        slots8 |= (uint64_t)sl << (8 * M);
        ++M;
      }
    }
    return M;
  };

  // shared expert gate/up: every row, act slot K
  {
    uint32_t rows4;
    uint64_t slots8;
    const int M = expert_rows(0, rows4, slots8);
    int c0, c1;
    Walk::sgu_range(p, c0, c1);
    for (int g = c0; g < c1; g += kCW) dispatch_gu(M, g, min(kCW, c1 - g), rows4, slots8);
  }
  trace(p, 6, ctid == 0);
  // routed gate/up: every compute warp must walk the same list, so one thread
  // takes the decision and the others read it after a barrier
  if (ctid == 0) {
    const bool ok = wait_flag(p, c, &c->lists_ready);
    c->nu_comp = (ok && !c->dead) ? c->nu : 0;
  }
  bar_sync(kBarCons, kCW * 32);
  const int nu = c->nu_comp;
  {
    long long g0, g1;
    Walk::rgu_range(p, nu, g0, g1);
    long long gch = g0;
    while (gch < g1) {
      const int u = (int)(gch / I), ch = (int)(gch % I);
      const int end = (int)min((long long)I, ch + (g1 - gch));
      uint32_t rows4;
      uint64_t slots8;
      const int M = expert_rows(u + 1, rows4, slots8);
      for (int g = ch; g < end; g += kCW) dispatch_gu(M, g, min(kCW, end - g), rows4, slots8);
      gch += end - ch;
    }
  }
  trace(p, 7, ctid == 0);
  // publish this CTA's activations, then wait for everyone's
  bar_sync(kBarCons, kCW * 32);
  if (ctid == 0) {
    __threadfence();
    red_release_add(&p.sync->cnt_act, 1u);
    wait_count(p, c, &p.sync->cnt_act, ep1 * (uint32_t)G, 4u);
  }
  int h0, h1;
  Walk::dn_range(p, h0, h1);
  const int nh = h1 - h0;
  for (int i = ctid; i < kMaxR * p.ymax; i += kCW * 32) ys[i] = 0.f;
  bar_sync(kBarCons, kCW * 32);
  trace(p, 8, ctid == 0);

  // ---------------- down projections, accumulated into ys [R][ymax]
  // Each expert's activation rows are staged in region A with cp.async; when
  // this expert's and the next one's rows both fit half of the region, the
  // next expert's rows are fetched while this one is computed.
  const size_t act_row_bytes = (size_t)I * 4;
  const size_t half_bytes = (size_t)(p.regA_bytes / 2) & ~(size_t)127;
  auto stage_act = [&](int x, uint8_t* dst) {
    uint32_t rows4;
    uint64_t slots8;
    const int M = expert_rows(x, rows4, slots8);
    const int per_row = I / 4;
    for (int i = ctid; i < M * per_row; i += kCW * 32) {
      const int t = i / per_row, k4 = i % per_row;
      const uint32_t r = (rows4 >> (4 * t)) & 15u, sl = (uint32_t)(slots8 >> (8 * t)) & 255u;
      cp_async16(dst + (size_t)t * act_row_bytes + (size_t)k4 * 16,
                 p.act + ((size_t)r * (K + 1) + sl) * I + (size_t)k4 * 4);
    }
    cp_async_commit();
  };
  auto m_of = [&](int x) -> int {
    if (x == 0) return R;
    return __popc(c->umask[x - 1]);
  };
  auto place = [&](int x) -> uint8_t* {
    return (size_t)m_of(x) * act_row_bytes <= half_bytes ? regA + (size_t)(x & 1) * half_bytes : regA;
  };
  bool prefetched = false;
  for (int x = 0; x <= nu; ++x) {
    uint32_t rows4;
    uint64_t slots8;
    const int M = expert_rows(x, rows4, slots8);
    uint8_t* act_s = place(x);
    if (!prefetched) {
      bar_sync(kBarCons, kCW * 32);   // everyone is done with the region's previous contents
      if (!c->dead) stage_act(x, act_s);
    }
    cp_async_wait_all();
    bar_sync(kBarCons, kCW * 32);     // this expert's rows are complete for every thread
    prefetched = x < nu && !c->dead && (size_t)M * act_row_bytes <= half_bytes &&
                 (size_t)m_of(x + 1) * act_row_bytes <= half_bytes;
    if (prefetched) stage_act(x + 1, place(x + 1));
    auto dn_group = [&](auto Mc, int g, int n) {
      constexpr int MM = decltype(Mc)::value;
      RowPtrs<MM> ar;
#pragma unroll
      for (int t = 0; t < MM; ++t) ar.p[t] = act_s + (size_t)t * act_row_bytes;
      float2 ad[MM];
#pragma unroll
      for (int t = 0; t < MM; ++t) ad[t] = make_float2(0.f, 0.f);
      const bool mine = warp < n;
      for (int k = 0; k < p.dn_nk; ++k) {
        const uint8_t* st = stage_wait(s);
        if (mine && !c->dead) dn_chunk<WT, MM>(st + (size_t)warp * p.dn_rc, p.dn_kc, k * p.dn_kc, ar, ad);
        stage_release(s);
        ++s;
      }
      if (mine) {
#pragma unroll
        for (int t = 0; t < MM; ++t) {
          const float d = warp_sum(ad[t].x + ad[t].y);
          if (lane == t) {
            const uint32_t r = (rows4 >> (4 * t)) & 15u, sl = (uint32_t)(slots8 >> (8 * t)) & 255u;
            const float wgt = x == 0 ? 1.0f : c->wt[r][sl];
            float* yp = ys + r * p.ymax + (g - h0) + warp;
            *yp = fmaf(wgt, d, *yp);
          }
        }
      }
    };
    for (int g = h0; g < h1; g += kCW) {
      const int n = min(kCW, h1 - g);
      switch (M) {
        case 1: dn_group(std::integral_constant<int, 1>{}, g, n); break;
        case 2: dn_group(std::integral_constant<int, 2>{}, g, n); break;
        case 3: dn_group(std::integral_constant<int, 3>{}, g, n); break;
        case 4: dn_group(std::integral_constant<int, 4>{}, g, n); break;
        case 5: dn_group(std::integral_constant<int, 5>{}, g, n); break;
        case 6: dn_group(std::integral_constant<int, 6>{}, g, n); break;
        case 7: dn_group(std::integral_constant<int, 7>{}, g, n); break;
        default: dn_group(std::integral_constant<int, 8>{}, g, n); break;
      }
    }
  }
  bar_sync(kBarCons, kCW * 32);
  trace(p, 9, ctid == 0);

  // ---------------- tail: y -> bf16, then the expand (or leave it pending)
  {
    // the Sinkhorn result is written by the control warps before they publish the lists
    const void* X = p.first ? p.x_prev : (const void*)p.xbuf;
    float* pend_y = p.pend_out + R * kS + R * kS * kS;
    for (int i = ctid; i < R * nh; i += kCW * 32) {
      const int r = i / nh, hh = i % nh, h = h0 + hh;
      float y = ys[r * p.ymax + hh];
      if (p.round_bf16) y = round_bf16(y);
      if (p.taps.y) p.taps.y[(size_t)r * H + h] = y;
      if (!p.last) {
        pend_y[(size_t)r * H + h] = y;
      } else {
#pragma unroll
        for (int si = 0; si < kS; ++si) {
          float acc = 0.f;
#pragma unroll
          for (int j = 0; j < kS; ++j)
            acc = fmaf(c->comb[r][si * kS + j], load_x_cg(X, ((size_t)r * kS + j) * H + h, p.hc_bf16), acc);
          acc = fmaf(c->post[r][si], y, acc);
          store_x(p.hc_out, ((size_t)r * kS + si) * H + h, acc, p.hc_bf16);
        }
      }
    }
  }
  bar_sync(kBarCons, kCW * 32);
  trace(p, 10, ctid == 0);
  if (ctid == 0 && !c->dead) {
    __threadfence();
    const uint32_t old = atomicAdd(&p.sync->cnt_done, 1u);
    if (old == ep1 * (uint32_t)G - 1u) {
      __threadfence();
      atomicAdd(&p.sync->epoch, 1u);
    }
  }
}

}  // namespace mono
