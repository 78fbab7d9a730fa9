// Quantised experts (FP8 e4m3 with 1 x 128 block scales, MXFP4) on the
// tensor cores: tcgen05.mma of kind::f8f6f4.  FP8 needs no conversion pass:
// the MMAs read the e4m3 weight codes straight from the ring (A, in shared
// memory), and the activations as e4m3 as well (B).
//
// An activation vector y goes into B as two e4m3 terms after a power-of-two
// scale 2^e that puts its largest magnitude in [128, 256): hi = e4m3(y 2^e)
// and lo = e4m3(y 2^e - hi).  B rows 0-7 carry hi of the 8 token rows, rows
// 8-15 lo; the epilogue adds the two halves of the accumulator and multiplies
// by 2^-e (exact).  A bf16 value has 8 significant bits and hi and lo hold 4
// each, so n (bf16) is represented exactly down to 2^-9 of its row's largest
// magnitude; smaller values, and the SwiGLU activations (fp32), keep an
// absolute error below 2^-10 of the scaled unit, about 2^-17 of the block's
// largest magnitude.
//   gate/up B: n, one scale per token row
//   down B:    the activations, one scale per (token row, 128-block of I),
//              chosen by the epilogue that completes the gate/up block and
//              stored behind the expert's codes
// The FP8 block scales (fp32, one per 1 x 128 block of a weight row) scale
// each unit's fp32 tile in the epilogue, so every unit gets its own
// accumulator (four in flight).
//
// Packed FP8 units: [8 chunks][128 rows][16]
// e4m3, chunk j of row i at [j][i]: K-major core matrices of 8 rows x 16
// bytes, 2048 bytes between K-neighbours and 128 between row groups.  A ring
// stage is one gate/up unit (gate, then up) or two down units, 32 KB.
//
// MXFP4 runs block-scaled MMAs (tcgen05.mma kind::mxf8f6f4.block_scale, e2m1
// A, e4m3 B, e8m0 scale factors): the weights' own 32-element block scales
// are applied inside the tensor core, so the codes go from HBM to the tensor
// core untouched.  A 2-D tensor map of the packed codes (data type
// 16U4_ALIGN16B) lets the TMA unit place each 16-code group in a 16-byte
// slot of shared memory (8 bytes of codes, 8 unused) with the 128-byte
// swizzle, which is the layout the MMA reads e2m1 from; a unit-matrix is 8 KB
// in HBM and 16 KB in the ring.  Its 4 x 128 scales (512 bytes, packed in the
// order tcgen05.cp expects) come with the same stage; the issuing lane copies
// them into tensor memory (tcgen05.cp 32x128b to all four lane quarters)
// right before the unit's MMAs, which pick the K-block's byte through the
// scale-factor id.  B's scale factors are all 1 (e8m0 127), written once:
// the activations keep their power-of-two row scales in the epilogue, as
// for FP8.
// Packed MXFP4 unit-matrices: 128 rows x 64 bytes row-major, gate/up units as
// (gate, up) pairs; scale chunks of 512 bytes in arrays of their own.
#pragma once
#include <cuda_fp8.h>

#include "tc_kernel.cuh"

namespace mono {

// one 128 x 128 unit of one matrix: bytes in HBM
template <int WT> struct TqFmt;
template <> struct TqFmt<W_FP8> {
  static constexpr int MAT_BYTES = 16384;
};
template <> struct TqFmt<W_FP4> {
  static constexpr int MAT_BYTES = 8192;
};

constexpr int kF8TmemCols = 128;   // four accumulators of 32 columns (gate 16 | up 16)
constexpr int kF4TmemCols = 256;   // the accumulators, then the scale factors
constexpr uint32_t kF4SfaCol = 128;   // A scale factors: 8 columns per ring slot (gate 4 | up 4, or 2 down units)
constexpr uint32_t kF4SfbNCol = 160;  // B scale factors of n (gate/up): 4 columns
constexpr uint32_t kF4SfbDnCol = 192; // B scale factors of a down expert's activations: I / 128 columns
constexpr int kF4MaxSlots = 4;        // ring slots whose A scales fit in tensor memory
constexpr int kF4MaxI = (kF4TmemCols - (int)kF4SfbDnCol) * 128;   // one down-scale column per 128 of I
constexpr int kF4Sf = 512;         // one scale chunk (tcgen05.cp 32x128b source)
constexpr int kF4SmemMat = 16384;  // one MXFP4 unit-matrix in the ring (16-byte slot per 16 codes)
constexpr int kF4SfOff = 2 * kF4SmemMat;   // the scale chunks of a stage, after its two unit-matrices
// transaction bytes one unit-matrix box of the tensor map counts on its
// mbarrier: the bytes of codes it writes (the 8-byte gaps of the 16-byte
// slots are left as they were, and the MMA does not read them)
constexpr uint32_t kF4BoxTx = kF4SmemMat / 2;
constexpr uint32_t kF8Acc = 4;
static_assert(kF8Acc <= (uint32_t)kMaxAcc, "accumulator barriers");
static_assert(kF4SfaCol + 8 * kF4MaxSlots <= kF4SfbNCol && kF4SfbNCol + 4 <= kF4SfbDnCol, "tensor memory");

// MXFP8 activations (act_mx8): one e4m3 term per token row (B has N = 8 rows)
// with an e8m0 scale per 32 values; tensor memory: 2 accumulators [0, 64), A
// scales 8 columns per ring slot [64, 96), B scales one 4-column group per
// 128 of the contraction from 96 (n's in the gate/up phase, a down expert's
// activations in the down phase).
constexpr uint32_t kMx8Acc = 2;
constexpr uint32_t kMx8SfaCol = 64;
constexpr uint32_t kMx8SfbCol = 96;
constexpr int kMx8MaxK = (kF4TmemCols - (int)kMx8SfbCol) / 4 * 128;   // 40 groups: 5120
static_assert(kMx8SfaCol + 8 * kF4MaxSlots <= kMx8SfbCol, "tensor memory");
// a down expert's operand: codes [I/16][8 rows][16], then one 512-byte scale
// chunk per 128 of I (lane n = row, byte j = 32-block j)
__host__ __device__ inline size_t mx8_act_stride(int I) { return (size_t)I * 8 + (size_t)(I / 128) * kF4Sf; }

// The e8m0 exponent X of a block of MXFP8 values (OCP MX rule: floor(log2
// amax) - 8, at least -127), from amax as fp32 bits; 0 codes for amax = 0.
__device__ __forceinline__ int mx8_exp(uint32_t amax_bits) {
  const int e = (int)((amax_bits >> 23) & 0xFFu);
  if (e == 0) return -127;              // zero or subnormal amax: the smallest scale
  return max(-127, e - 127 - 8);
}

// bytes of one expert entry's down B operand: [I/16][16 rows][16] e4m3 codes,
// then [I/128][8] fp32 inverse scales; with MXFP4 (block-scaled MMAs) also
// the same scales as e8m0 B scale factors, one 512-byte chunk per 4 blocks:
// lane n (B row, < 16) byte j of chunk g = the scale of block 4 g + j
__host__ __device__ inline size_t f8_act_stride(int I, bool mx) {
  return (size_t)I * 16 + (size_t)(I / 128) * 32 + (mx ? (size_t)(I / 512) * kF4Sf : 0);
}

// e with m 2^e in [128, 256) for m > 0 (0 for m = 0), within [-126, 126] so
// that 2^e and 2^-e are normal floats
__device__ __forceinline__ int f8_exp(float m) {
  if (!(m > 0.f)) return 0;
  const int ex = (int)((__float_as_uint(m) >> 23) & 0xFFu) - 127;   // floor(log2 m) for normal m
  return max(-126, min(126, 7 - ex));
}
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// two scaled values -> e4m3 hi and lo code pairs (the first value in the low byte)
__device__ __forceinline__ void f8_split2(float y0, float y1, uint32_t& hi, uint32_t& lo) {
  const __nv_fp8x2_storage_t h = __nv_cvt_float2_to_fp8x2(make_float2(y0, y1), __NV_SATFINITE, __NV_E4M3);
  const float2 hf = __half22float2(__half2(__nv_cvt_fp8x2_to_halfraw2(h, __NV_E4M3)));
  const __nv_fp8x2_storage_t l =
      __nv_cvt_float2_to_fp8x2(make_float2(y0 - hf.x, y1 - hf.y), __NV_SATFINITE, __NV_E4M3);
  hi = h;
  lo = l;
}

// n, bf16 in the layout [H/8][8 rows][8], becomes the e4m3 B operand
// [H/16][16 rows][16] (rows 0-7 hi, 8-15 lo) in place, one 128-column block
// per warp at a time (the two layouts put a block in the same 2 KB); c->nsc
// gets each row's inverse scale.  Compute warps.
__device__ void f8_convert_n(const Params& p, Ctl* c, uint8_t* regA) {
  const int H = p.H, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // row maxima: 16-byte item q of the bf16 layout holds row q & 7, and this
  // thread's items all have row tid & 7
  float m = 0.f;
  for (int q = tid; q < H; q += kCW * 32) {
    const uint4 v = *reinterpret_cast<const uint4*>(regA + (size_t)q * 16);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(v.x)), fabsf(bf16hi(v.x))), fmaxf(fabsf(bf16lo(v.y)), fabsf(bf16hi(v.y)))));
    m = fmaxf(m, fmaxf(fmaxf(fabsf(bf16lo(v.z)), fabsf(bf16hi(v.z))), fmaxf(fabsf(bf16lo(v.w)), fabsf(bf16hi(v.w)))));
  }
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 16));
  if (lane < 8) c->sq[warp][lane] = m;
  bar_sync(kBarCons, kCW * 32);
  const int r = lane & 7, q = lane >> 3;
  float mr = 0.f;
#pragma unroll
  for (int w = 0; w < kCW; ++w) mr = fmaxf(mr, c->sq[w][r]);
  const int e = f8_exp(mr);
  if (tid < 8) c->nsc[tid] = pow2i(-e);
  const float sc = pow2i(e);
  // lane (r, q): columns 32 q .. 32 q + 31 of row r of the block, i.e. bf16
  // chunks 4q .. 4q + 3 in, e4m3 chunks 2q and 2q + 1 out
  for (int kb = warp; kb < H / 128; kb += kCW) {
    uint8_t* blk = regA + (size_t)kb * 2048;
    uint4 v[4];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) v[cc] = *reinterpret_cast<const uint4*>(blk + (4 * q + cc) * 128 + r * 16);
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int m2 = 0; m2 < 4; ++m2) {
        const uint4 s = v[2 * h + (m2 >> 1)];
        const uint32_t w0 = (m2 & 1) ? s.z : s.x, w1 = (m2 & 1) ? s.w : s.y;
        uint32_t h01, l01, h23, l23;
        f8_split2(bf16lo(w0) * sc, bf16hi(w0) * sc, h01, l01);
        f8_split2(bf16lo(w1) * sc, bf16hi(w1) * sc, h23, l23);
        hi[m2] = h01 | (h23 << 16);
        lo[m2] = l01 | (l23 << 16);
      }
      *reinterpret_cast<uint4*>(blk + (2 * q + h) * 256 + r * 16) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(blk + (2 * q + h) * 256 + (8 + r) * 16) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
  }
}

// n, bf16 in the layout [H/8][8 rows][8], becomes MXFP8: e4m3 codes
// [H/16][8 rows][16] in place (the B operand of N = 8), and one e8m0 scale
// per (row, 32 columns) into sf[unit][row] (4 bytes: the unit's 32-blocks)
// for the tensor-memory copy.  Lane (r, q) of a warp takes columns 32q ..
// 32q + 31 of row r of a 128-column block: exactly one 32-block, so its
// scale needs no exchange.  Blocks go in waves of one per warp; a wave
// reads all its inputs before any output is written, and a block's output
// (1 KB at kb KB) only overlaps the input of block kb / 2, which an earlier
// wave (or this one, before its barrier) has read.  Compute warps.
__device__ void mx8_convert_n(const Params& p, uint8_t* regA, uint32_t* sf) {
  const int H = p.H, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = lane & 7, q = lane >> 3, nb = H / 128;
  for (int kb0 = 0; kb0 < nb; kb0 += kCW) {
    const int kb = kb0 + warp;
    uint4 v[4];
    if (kb < nb) {
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) v[cc] = *reinterpret_cast<const uint4*>(regA + (size_t)(kb * 16 + 4 * q + cc) * 128 + r * 16);
    }
    bar_sync(kBarCons, kCW * 32);
    if (kb < nb) {
      float x[32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        x[8 * cc + 0] = bf16lo(v[cc].x); x[8 * cc + 1] = bf16hi(v[cc].x);
        x[8 * cc + 2] = bf16lo(v[cc].y); x[8 * cc + 3] = bf16hi(v[cc].y);
        x[8 * cc + 4] = bf16lo(v[cc].z); x[8 * cc + 5] = bf16hi(v[cc].z);
        x[8 * cc + 6] = bf16lo(v[cc].w); x[8 * cc + 7] = bf16hi(v[cc].w);
      }
      float m = 0.f;
#pragma unroll
      for (int k = 0; k < 32; ++k) m = fmaxf(m, fabsf(x[k]));
      const int X = mx8_exp(__float_as_uint(m));
      const float inv = pow2i(-X);   // X <= 120 for finite bf16 values, so 2^-X is a normal float
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x[4 * k] * inv, x[4 * k + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(x[4 * k + 2] * inv, x[4 * k + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        w[k] = lo | (hi << 16);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h)
        *reinterpret_cast<uint4*>(regA + (size_t)(kb * 8 + 2 * q + h) * 128 + r * 16) =
            make_uint4(w[4 * h], w[4 * h + 1], w[4 * h + 2], w[4 * h + 3]);
      reinterpret_cast<uint8_t*>(sf)[((size_t)kb * 8 + r) * 4 + q] = m > 0.f ? (uint8_t)(X + 127) : (uint8_t)0;
    }
    bar_sync(kBarCons, kCW * 32);
  }
}

// A complete gate/up block: SwiGLU, then each token row's 128 activations of
// the block as e4m3 hi/lo under the block's power-of-two scale, into the
// down B operand of expert entry x, with the inverse scale behind the codes;
// zero for rows that do not use the expert.  Then the block counts for its
// expert.  Every epilogue thread, live or not.
__device__ __forceinline__ void f8_store_act(const Params& p, Ctl* c, const Seg& sg, bool live, int i,
                                             const float (&a)[8], const float (&b)[8], bool mx) {
  const int R = p.R, K = p.K, I = p.I, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int x = sg.x;
  float act[8];
#pragma unroll
  for (int r = 0; r < kMaxR; ++r) {
    const int sl = x == 0 ? K : c->uslot[x - 1][r];
    act[r] = 0.f;
    if (live && r < R && sl >= 0) {
      float gg = a[r], uu = b[r];
      if (p.round_bf16) {
        gg = round_bf16(gg);
        uu = round_bf16(uu);
      }
      act[r] = gg / (1.0f + expf(-gg)) * uu;
    }
    const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(act[r])));
    if (lane == 0) c->amax[warp][r] = __uint_as_float(mb);
  }
  bar_sync(kBarEpi, 4 * 32);
  uint8_t* base = p.actb + (size_t)x * f8_act_stride(I, mx);
  const int ch = sg.blk * 128 + i;
  uint8_t* dst = base + (size_t)(ch >> 4) * 256 + (ch & 15);
#pragma unroll
  for (int r = 0; r < kMaxR; r += 2) {
    int e[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int rr = r + k;
      e[k] = f8_exp(fmaxf(fmaxf(c->amax[0][rr], c->amax[1][rr]), fmaxf(c->amax[2][rr], c->amax[3][rr])));
    }
    uint32_t hb, lb;
    f8_split2(act[r] * pow2i(e[0]), act[r + 1] * pow2i(e[1]), hb, lb);
    if (live) {
      dst[r * 16] = (uint8_t)(hb & 0xFFu);
      dst[(r + 1) * 16] = (uint8_t)(hb >> 8);
      dst[(8 + r) * 16] = (uint8_t)(lb & 0xFFu);
      dst[(9 + r) * 16] = (uint8_t)(lb >> 8);
      float* inv = reinterpret_cast<float*>(base + (size_t)I * 16) + sg.blk * 8;
      if (i == r) inv[r] = pow2i(-e[0]);
      if (i == r + 1) inv[r + 1] = pow2i(-e[1]);
      if (mx && (i == r || i == r + 1)) {
        // the block's scale as the e8m0 B scale factor of rows rr (hi) and
        // 8 + rr (lo): byte (blk % 4) of lane n in chunk blk / 4
        const int rr = i;
        const uint8_t code = (uint8_t)(127 - e[rr - r]);
        uint8_t* sfb = base + (size_t)I * 16 + (size_t)(I / 128) * 32 + (size_t)(sg.blk / 4) * kF4Sf + (sg.blk % 4);
        sfb[16 * rr] = code;
        sfb[16 * (8 + rr)] = code;
      }
    }
  }
  // the block's activations are out: count it for its expert (the codes are
  // read by a bulk copy, the async proxy; the scales by the epilogues)
  __threadfence();
  bar_sync(kBarEpi, 4 * 32);   // reached by every epilogue thread, live or not
  if (tid == 0 && live && may_publish(p, c->epoch, 0, 8) && !(p.fault_stage == 4 && x == 0 && sg.blk == 0)) {
    fence_proxy_async_global();
    red_release_add(&p.xready[x], 1u);
  }
}

// MXFP8 activations: a complete gate/up block's SwiGLU as e4m3 codes of the
// down B operand [I/16][8 rows][16] of expert entry x, each token row's 32
// channels of a warp under their own e8m0 scale (OCP MX rule), the scale
// byte at lane r, byte = warp, of the block's 512-byte chunk; zero for rows
// that do not use the expert.  Then the block counts for its expert.  Every
// epilogue thread, live or not.
__device__ __forceinline__ void mx8_store_act(const Params& p, Ctl* c, const Seg& sg, bool live, int i,
                                              const float (&a)[8], const float (&b)[8]) {
  const int R = p.R, K = p.K, I = p.I, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int x = sg.x;
  uint8_t* base = p.actb + (size_t)x * mx8_act_stride(I);
  const int ch = sg.blk * 128 + i;
  uint8_t* dst = base + (size_t)(ch >> 4) * 128 + (ch & 15);
  uint8_t* sfc = base + (size_t)I * 8 + (size_t)sg.blk * kF4Sf;
#pragma unroll
  for (int r = 0; r < kMaxR; ++r) {
    const int sl = x == 0 ? K : c->uslot[x - 1][r];
    float act = 0.f;
    if (live && r < R && sl >= 0) {
      float gg = a[r], uu = b[r];
      if (p.round_bf16) {
        gg = round_bf16(gg);
        uu = round_bf16(uu);
      }
      act = gg / (1.0f + expf(-gg)) * uu;
    }
    const uint32_t mb = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(act)));
    const int X = mx8_exp(mb);
    const uint32_t code = __nv_cvt_float2_to_fp8x2(make_float2(act * pow2i(-X), 0.f), __NV_SATFINITE, __NV_E4M3);
    if (live) {
      dst[r * 16] = (uint8_t)(code & 0xFFu);
      if (lane == 0) sfc[16 * r + warp] = mb ? (uint8_t)(X + 127) : (uint8_t)0;
    }
  }
  // the block's activations are out: count it for its expert (read by a
  // bulk copy, the async proxy)
  __threadfence();
  bar_sync(kBarEpi, 4 * 32);   // reached by every epilogue thread, live or not
  if (tid == 0 && live && may_publish(p, c->epoch, 0, 8) && !(p.fault_stage == 4 && x == 0 && sg.blk == 0)) {
    fence_proxy_async_global();
    red_release_add(&p.xready[x], 1u);
  }
}

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) mono_ffn_tq_kernel(const __grid_constant__ Params p) {
  constexpr bool F4 = WT == W_FP4;                    // block-scaled MMAs on e2m1 codes
  constexpr uint32_t MAT = TqFmt<WT>::MAT_BYTES;      // one unit of one matrix in HBM
  extern __shared__ __align__(1024) uint8_t smem[];
  const SmemLayout L(p.nst, p.slot_bytes, p.regA_bytes, p.ymax);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + p.nst;
  Ctl* c = reinterpret_cast<Ctl*>(smem + L.ctl);
  uint8_t* regA = smem + L.regA;   // n (gate/up B operand), then the down B operand
  uint8_t* ring = smem + L.ring;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int H = p.H, I = p.I, K = p.K, G = p.G;
  const TcGeo geo(p);

  // launched behind another grid of the stream (programmatic dependent
  // launch), this grid may be resident before that one has finished: nothing
  // it wrote is read before this point
  grid_dep_wait();
  if (threadIdx.x >= 32 && threadIdx.x < 64) {
    // this CTA's slice of the mix weights and of the residual streams to L2
    // while thread 0 sets up (the prologue's first loads then hit L2)
    const int lane = threadIdx.x & 31;
    int h0, h1;
    Walk::dn_range(p, h0, h1);
    const int nh = h1 - h0;
    for (int sg = lane; sg < kS; sg += 32)
      prefetch_l2_span(p.mix_w + ((size_t)sg * p.H + h0) * kMixC, (size_t)nh * kMixC * 4);
    const int eb = p.hc_bf16 ? 2 : 4;
    for (int q = lane; q < p.R * kS; q += 32) {
      const uint8_t* row = reinterpret_cast<const uint8_t*>(p.x_prev) + ((size_t)q * p.H + h0) * eb;
      for (int o = 0; o < nh * eb; o += 128) prefetch_l2_line(row + o);
      prefetch_l2_line(row + nh * eb - 1);
    }
  }
  if (tid == 0) {
    // both grid words in flight at once, used after the barrier set-up
    const uint32_t ep0 = ld_relaxed(&p.sync->cnt_done);
    const uint32_t abort0 = ld_relaxed(&p.err->abort);
    c->dead = 0;
    c->lists_ready = 0;
    c->nu = 0;
    c->n_ready = 0;
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);   // the MMAs' commit
    }
    for (uint32_t b = 0; b < kF8Acc; ++b) {
      mbar_init(&c->accfull[b], 1);
      mbar_init(&c->accempty[b], 4);
    }
    mbar_init(&c->drain, 1);
    mbar_init(&c->bfull, 1);
    c->epoch = ep0;
    c->live = live_rows(p);
    if (abort0) c->dead = 1;   // fail-stop after an unreported error
    fence_barrier_init();
  }
  __syncthreads();
  grid_dep_launch();   // the next layer's grid may take each SM as this grid leaves it
  if (c->dead) return;
  constexpr int kCols = F4 ? kF4TmemCols : kF8TmemCols;
  if (warp == kMmaWarp) tmem_alloc(&c->tmem_base, kCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t ep1 = c->epoch + (uint32_t)G;   // every grid counter's target in this launch
  const uint32_t tmem = c->tmem_base;
  trace(p, 0, tid == 0);

  // a ring stage: one gate/up unit (gate, up) or two down units
  auto stage_units = [&](const Seg& sg) { return sg.list != L_DN ? 1 : 2; };

  // ================================================================ producer
  if (warp == kProdWarp) {
    uint32_t s = 0, issued = 0;
    bool ok = true, dry = false;
    auto seg = [&](const Seg& sg) {
      if (lane != 0) return;
      const int e = seg_expert(p, c, sg.x);
      const bool gu = sg.list != L_DN;
      const int per = stage_units(sg);
      if (F4) {
        // unit-matrix m of the list's packed array: gate/up pairs (2 u, 2 u + 1)
        // of unit u, or down unit u; each a box of 128 rows of the tensor map
        const long long m0 = gu ? ((long long)(e * geo.nbi + sg.blk) * geo.upb_gu) * 2
                                : (long long)(e * geo.nbh + sg.blk) * geo.upb_dn;
        const CUtensorMap* map = gu ? &p.tm_gu : &p.tm_dn;
        const uint8_t* sf = reinterpret_cast<const uint8_t*>(gu ? p.gsc : p.dsc);
        for (int u = sg.k0; u < sg.k1; u += per) {
          const uint32_t slot = s % p.nst, q = s / p.nst;
          const int nm = gu ? 2 : min(per, sg.k1 - u);   // unit-matrices in this stage
          const long long m = gu ? m0 + 2 * u : m0 + u;
          if (ok && !dry && q > 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
          if (ok && !dry) {
            uint8_t* dst = ring + (size_t)slot * p.slot_bytes;
            mbar_arrive_expect_tx(&full[slot], (uint32_t)nm * (kF4BoxTx + kF4Sf));
            for (int j = 0; j < nm; ++j) tma_load_2d(dst + j * kF4SmemMat, map, 0, (int)((m + j) * 128), &full[slot]);
            tma_load_1d(dst + kF4SfOff, sf + m * kF4Sf, (uint32_t)nm * kF4Sf, &full[slot]);
            issued = s + 1;
          }
          ++s;
        }
        return;
      }
      const uint8_t* base = gu ? p.gu + (size_t)e * p.gu_estride + (size_t)sg.blk * geo.upb_gu * 2 * MAT
                               : p.dn + (size_t)e * p.dn_estride + (size_t)sg.blk * geo.upb_dn * MAT;
      const uint32_t ub = gu ? 2u * MAT : MAT;
      // the epilogue's FP8 block scales [unit][gate | up] or [unit] per block
      const uint32_t sc_unit = gu ? 256u : 128u;
      const float* sc_base = gu ? p.gsc + (size_t)(e * geo.nbi + sg.blk) * geo.upb_gu * 256
                                : p.dsc + (size_t)(e * geo.nbh + sg.blk) * geo.upb_dn * 128;
      for (int u = sg.k0; u < sg.k1; u += per) {
        const uint32_t slot = s % p.nst, q = s / p.nst;
        const uint32_t n = (uint32_t)min(per, sg.k1 - u), bytes = n * ub;
        if (ok && !dry && q > 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
        if (ok && !dry) {
          mbar_arrive_expect_tx(&full[slot], bytes);
          tma_load_1d(ring + (size_t)slot * p.slot_bytes, base + (size_t)u * ub, bytes, &full[slot]);
          issued = s + 1;
          prefetch_l2(sc_base + (size_t)u * sc_unit, n * sc_unit * 4);   // read by the epilogue
        }
        ++s;
      }
    };
    if (lane == 0) {
      const int e0 = (int)(blockIdx.x * (uint32_t)p.E / G), e1 = (int)((blockIdx.x + 1) * (uint32_t)p.E / G);
      if (!p.dense) prefetch_l2_span(p.router_t + (size_t)e0 * H, (size_t)(e1 - e0) * H * 4);
      prefetch_l2_span(p.norm_w, (size_t)H * (p.norm_bf16 ? 2 : 4));
      prefetch_l2_span(p.bias, (size_t)p.E * 4);
    }
    tc_segments(p, geo, L_SGU, 0, seg);
    {
      // the routed list's loop once with no waits or copies (one expert's
      // worth of stages, addresses never used), so that its code is in the
      // instruction cache when the lists arrive
      const uint32_t s0 = s;
      dry = true;
      tc_segments(p, geo, L_RGU, 1, seg);
      dry = false;
      s = s0;
    }
    if (ok && lane == 0) ok = wait_flag(p, c, &c->lists_ready);
    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    const int nu = ok ? *(volatile int*)&c->nu : 0;
    trace(p, 11, lane == 0);
    tc_segments(p, geo, L_RGU, nu, seg);
    tc_segments(p, geo, L_DN, nu, seg);
    trace(p, 12, lane == 0);
    if (lane == 0) {   // no bulk copy may still target this CTA's shared memory at exit
      const uint32_t first = issued > (uint32_t)p.nst ? issued - p.nst : 0;
      for (uint32_t t = first; t < issued; ++t) {
        const uint64_t t0 = globaltimer();
        while (!mbar_test(&full[t % p.nst], (t / p.nst) & 1)) {
          if (globaltimer() - t0 > p.timeout_ns) break;
          __nanosleep(64);
        }
      }
    }
    return;
  }

  // =========================================================== MMA issuer
  if (warp == kMmaWarp) {
    uint32_t s = 0, t = 0, ndrain = 0, nb = 0;
    int prev_x = -1;
    bool first_rgu = true, b_pending = false;
    auto warp_ok = [&](bool v) { return __shfl_sync(0xffffffffu, (int)v, 0) != 0; };
    bool ok = true;
    if (lane == 0) ok = wait_flag(p, c, &c->n_ready);
    ok = warp_ok(ok);
    const bool mx8 = F4 && p.mx8;
    const uint32_t nacc = mx8 ? kMx8Acc : kF8Acc;
    const uint32_t idesc =
        F4 ? umma_idesc_mx_e2m1_e4m3(128, mx8 ? 8 : 16) : umma_idesc_e4m3(128, 16);
    // the down B operand: codes, and for MXFP4 also its e8m0 scale chunks
    // (the fp32 inverse scales between them are read by the epilogue only)
    const uint32_t b_bytes = mx8 ? (uint32_t)mx8_act_stride(I) : F4 ? (uint32_t)f8_act_stride(I, true) : (uint32_t)I * 16u;
    // B (n, or a down expert's activations): [K/16][16 rows][16], 256 bytes
    // between K-neighbours, rows 8-15 128 bytes on, a unit 2048 bytes; with
    // MXFP8 activations [K/16][8 rows][16]: 128 bytes between K-neighbours, a
    // unit 1024 bytes
    const uint64_t bdesc = mx8 ? umma_desc(smem_u32(regA), 128u, 128u) : umma_desc(smem_u32(regA), 256u, 128u);
    const uint32_t bunit = mx8 ? 64u : 128u, bkstep = mx8 ? 16u : 32u;   // descriptor units per unit / K-step
    auto seg = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      if (!gu && sg.x != prev_x) {
        // a new down expert: its activations complete, every MMA on the B
        // region done, then one bulk copy of this expert's operand
        if (lane == 0 && ok) ok = wait_count(p, c, &p.xready[sg.x], (uint32_t)geo.nbi, 4u);
        ok = warp_ok(ok);
        fence_proxy_async_global();
        trace(p, 8, prev_x < 0 && lane == 0);
        umma_commit_warp(&c->drain);
        if (lane == 0 && ok) ok = wait_bar(p, c, &c->drain, ndrain & 1u);
        ok = warp_ok(ok);
        ++ndrain;
        tc_fence_after();
        prev_x = sg.x;
        if (ok) {   // (a copy whose wait failed is waited for again at exit)
          if (lane == 0) {
            mbar_arrive_expect_tx(&c->bfull, b_bytes);
            tma_load_1d(regA, p.actb + (size_t)sg.x * (mx8 ? mx8_act_stride(I) : f8_act_stride(I, F4)), b_bytes,
                        &c->bfull);
            ok = wait_bar(p, c, &c->bfull, nb & 1u);
          }
          ok = warp_ok(ok);
          b_pending = !ok;
          ++nb;
        }
        tc_fence_after();
        if (mx8 && ok) {
          // the expert's activation scales: unit u's chunk to the 4-column
          // group from kMx8SfbCol + 4u (n's scales there are no longer read:
          // the drain above completed every gate/up MMA)
          const uint8_t* sfb = regA + (size_t)I * 8;
          for (int u = 0; u < I / 128; ++u)
            tmem_cp_sf(tmem + kMx8SfbCol + 4u * u, umma_desc(smem_u32(sfb + (size_t)u * kF4Sf), 16u, 128u));
        } else if (F4 && ok) {
          // the expert's activation scales: chunk g (blocks 4 g .. 4 g + 3)
          // to the 4 B-scale columns from kF4SfbDnCol + 4 g
          const uint8_t* sfb = regA + (size_t)I * 16 + (size_t)(I / 128) * 32;
          for (int g = 0; g < I / 512; ++g)
            tmem_cp_sf(tmem + kF4SfbDnCol + 4u * g, umma_desc(smem_u32(sfb + (size_t)g * kF4Sf), 16u, 128u));
        }
        trace(p, 15, nb == 1 && lane == 0);
      }
      const int per = stage_units(sg);
      if (F4) {
        // MXFP4: the weights' block scales and the activations' scales are
        // applied inside the MMAs, so the whole segment accumulates in one
        // buffer.  Stage s's A scale chunks go to the 8 columns of its ring
        // slot (gate 4 | up 4, or unit 0 | unit 1), free again once the
        // slot's MMAs are complete (which the producer waits for).
        const uint32_t buf = t % nacc;
        if (t >= nacc) {
          if (lane == 0 && ok) ok = wait_bar(p, c, &c->accempty[buf], ((t / nacc) - 1) & 1u);
          ok = warp_ok(ok);
        }
        tc_fence_after();
        for (int u0 = sg.k0; u0 < sg.k1; u0 += per) {
          const uint32_t slot = s % p.nst, q = s / p.nst;
          const int n = min(per, sg.k1 - u0);
          if (lane == 0 && ok) ok = wait_bar(p, c, &full[slot], q & 1);
          ok = warp_ok(ok);
          tc_fence_after();
          if (sg.list == L_RGU && first_rgu) {
            first_rgu = false;
            trace(p, 13, lane == 0);
          }
          const uint8_t* a_st = ring + (size_t)slot * p.slot_bytes;
          const uint32_t sfa = tmem + (mx8 ? kMx8SfaCol : kF4SfaCol) + 8u * slot;
          for (int j = 0; j < n && ok; ++j) {
            const int u = u0 + j;
            const uint8_t* a = a_st + (size_t)j * kF4SmemMat;   // gate/up: gate here, up 16 KB on
            const uint8_t* sf = a_st + kF4SfOff + j * kF4Sf;
            // B scales.  MXFP8 activations: unit u's group, byte = K-block.
            // Otherwise gate/up: n's scale per row (any byte); down: unit u's
            // scale, byte u % 4 of the columns of its chunk
            const uint32_t sfb = mx8 ? tmem + kMx8SfbCol + 4u * (uint32_t)u
                                     : gu ? tmem + kF4SfbNCol : tmem + kF4SfbDnCol + 4u * (uint32_t)(u / 4);
            const bool bstep = mx8 || gu;
            umma_unit_mx(tmem + 32u * buf, umma_desc_sw128(smem_u32(a), 1024u), bdesc + (uint64_t)(u * bunit), bkstep,
                         idesc, sfa + 4u * j, umma_desc(smem_u32(sf), 16u, 128u), sfa + 4u,
                         umma_desc(smem_u32(sf + kF4Sf), 16u, 128u), sfb, bstep, bstep ? 0u : (uint32_t)(u % 4),
                         u > sg.k0, gu);
          }
          umma_commit_warp(&empty[slot]);
          ++s;
        }
        umma_commit_warp(&c->accfull[buf]);
        ++t;
        return;
      }
      for (int u0 = sg.k0; u0 < sg.k1; u0 += per) {
        // the stage's A in the ring slot: FP8 unit-matrices of 16 KB in the
        // no-swizzle core-matrix layout
        const uint32_t slot = s % p.nst, q = s / p.nst;
        const int n = min(per, sg.k1 - u0);
        if (lane == 0 && ok) ok = wait_bar(p, c, &full[slot], q & 1);
        ok = warp_ok(ok);
        tc_fence_after();
        const uint8_t* a_st = ring + (size_t)slot * p.slot_bytes;
        if (sg.list == L_RGU && first_rgu) {
          first_rgu = false;
          trace(p, 13, lane == 0);
        }
        for (int j = 0; j < n; ++j) {
          const int u = u0 + j;
          const uint32_t buf = t % kF8Acc;
          if (t >= kF8Acc) {
            if (lane == 0 && ok) ok = wait_bar(p, c, &c->accempty[buf], ((t / kF8Acc) - 1) & 1u);
            ok = warp_ok(ok);
          }
          tc_fence_after();
          if (ok) {
            const uint64_t da = umma_desc(smem_u32(a_st + (size_t)j * MAT), 2048u, 128u);
            umma_unit_e4m3(tmem + 32u * buf, da, bdesc + (uint64_t)(u * 128), 32u, idesc, gu);
          }
          umma_commit_warp(&c->accfull[buf]);
          ++t;
        }
        umma_commit_warp(&empty[slot]);
        ++s;
      }
    };
    tc_segments(p, geo, L_SGU, 0, seg);
    if (lane == 0 && ok) ok = wait_flag(p, c, &c->lists_ready);
    ok = warp_ok(ok);
    const int nu = ok ? *(volatile int*)&c->nu : 0;
    tc_segments(p, geo, L_RGU, nu, seg);
    trace(p, 14, lane == 0);
    tc_segments(p, geo, L_DN, nu, seg);
    trace(p, 16, lane == 0);
    // every MMA of this CTA is complete before the tensor memory goes away,
    // and no bulk copy still targets shared memory at exit
    umma_commit_warp(&c->drain);
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_test(&c->drain, ndrain & 1u) && globaltimer() - t0 < p.timeout_ns) __nanosleep(64);
      while (b_pending && !mbar_test(&c->bfull, (nb - 1) & 1u) && globaltimer() - t0 < 2 * p.timeout_ns)
        __nanosleep(64);
    }
    __syncwarp();
    bar_sync(kBarEnd, 5 * 32);
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
    return;
  }

  // ================================================================ prologue
  prologue_mix(p, c, regA, ep1);
  if (warp >= kCtlWarp0) {
    control_warps(p, c, regA, ep1, false, p.R <= 4);
    return;
  }
  collapse_norm<true>(p, c, regA, ep1);
  // the router reads n as bf16 (the layer's values); the MMAs then take it
  // as e4m3 hi/lo
  router_logits<true>(p, c, regA, false);
  const bool mx8 = F4 && p.mx8;
  uint32_t* mx8_sf = reinterpret_cast<uint32_t*>(c->red);   // [H/128][8] scale words of n (the prologue is done with red)
  if (mx8) mx8_convert_n(p, regA, mx8_sf);
  else f8_convert_n(p, c, regA);
  fence_proxy_async_smem();   // n is read by the tensor cores (async proxy)
  bar_sync(kBarCons, kCW * 32);
  if (mx8 && warp < 4) {
    // n's scales as the B scale factors of the gate/up MMAs: 128-unit u in
    // the 4-column group from kMx8SfbCol + 4u, lane n = row, byte j = its
    // 32-block j, in every lane quarter
    const uint32_t tq = tmem + ((uint32_t)(warp * 32) << 16) + kMx8SfbCol;
    for (int u = 0; u < H / 128; ++u)
      tmem_st4(tq + 4u * u, lane < 8 ? mx8_sf[u * 8 + lane] : 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu);
    tmem_st_wait();
    tc_fence_before();
  }
  if (F4 && !mx8 && warp < 4) {
    // n's row scales as the B scale factors of the gate/up MMAs: lane n of
    // every lane quarter holds B row n's e8m0 code (rows 8-15, the lo terms,
    // share their token row's scale) in every byte of its first column
    const uint32_t code = lane < 16 ? (__float_as_uint(c->nsc[lane & 7]) >> 23) & 0xFFu : 127u;
    tmem_st4(tmem + ((uint32_t)(warp * 32) << 16) + kF4SfbNCol, code * 0x01010101u, 0x7F7F7F7Fu, 0x7F7F7F7Fu,
             0x7F7F7F7Fu);
    tmem_st_wait();
    tc_fence_before();
  }
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) *(volatile int*)&c->n_ready = 1;
  trace(p, 3, tid == 0);
  // R <= 4: warps 4-7 take the top-k while warps 0-3 start on the shared
  // expert's tiles, which need no routing
  const bool split = p.R <= 4;
  if (!split || warp >= 4) route_rows(p, c, ep1, split);
  // the warps that need it agree on the expert list once
  int nu = 0;
  auto agree = [&]() {
    if (tid == 0) {
      const bool ok = wait_flag(p, c, &c->lists_ready);
      c->nu_comp = (ok && !c->dead) ? c->nu : 0;
    }
  };
  if (!split) {
    agree();
    bar_sync(kBarCons, kCW * 32);
    nu = c->nu_comp;
  }

  if (warp < 4) {
    // ============================================================ epilogue
    // thread <-> row i = 32 w + l of the 128-row tile (its TMEM lane)
    const int i = tid;
    uint32_t t = 0;
    bool ok = true;
    const uint32_t nacc = mx8 ? kMx8Acc : kF8Acc;
    auto take = [&](uint32_t* v, uint32_t* w2, bool gu) {   // the next unit's (or MXFP4 segment's) tile
      const uint32_t buf = t % nacc;
      if (ok) ok = wait_bar(p, c, &c->accfull[buf], (t / nacc) & 1u);
      tc_fence_after();
      const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16) + 32u * buf;
      tmem_ld16(ta, v);
      if (gu) tmem_ld16(ta + 16u, w2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c->accempty[buf]);
      ++t;
    };
    auto seg = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      const int upb = gu ? geo.upb_gu : geo.upb_dn;
      const int e = seg_expert(p, c, sg.x);
      float a[8], b[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = b[r] = 0.f;
      uint32_t v[16], w2[16];
      if (F4) {
        // the segment's sums, every scale already applied in the MMAs: the
        // hi (rows 0-7) and lo (rows 8-15) columns of each token row added
        take(v, w2, gu);
#pragma unroll
        for (int r = 0; r < 8; ++r) {   // MXFP8 activations: one term (N = 8)
          a[r] = mx8 ? __uint_as_float(v[r]) : __uint_as_float(v[r]) + __uint_as_float(v[8 + r]);
          b[r] = !gu ? 0.f : mx8 ? __uint_as_float(w2[r]) : __uint_as_float(w2[r]) + __uint_as_float(w2[8 + r]);
        }
        trace(p, 20, t == 1 && tid == 0);
        const bool live = ok && !c->dead;
        if (!epi_combine(p, c, geo, sg, upb, gu, live, i, a, b)) return;
        if (gu && mx8) mx8_store_act(p, c, sg, live, i, a, b);
        else if (gu) f8_store_act(p, c, sg, live, i, a, b, true);
        else epi_store(p, c, geo, sg, false, live, i, a, b);
        return;
      }
      // the units' FP8 block scales (brought to L2 by the producer), two units
      // ahead; MXFP4 block scales are applied inside the MMA (1 here)
      const float* sc = gu ? p.gsc + (size_t)(e * geo.nbi + sg.blk) * upb * 256
                           : p.dsc + (size_t)(e * geo.nbh + sg.blk) * upb * 128;
      const int us = gu ? 256 : 128;
      auto ld_g = [&](int u) { return F4 ? 1.f : u < sg.k1 ? __ldg(sc + (size_t)u * us + i) : 0.f; };
      auto ld_u = [&](int u) { return F4 ? 1.f : gu && u < sg.k1 ? __ldg(sc + (size_t)u * us + 128 + i) : 0.f; };
      float sg0 = ld_g(sg.k0), su0 = ld_u(sg.k0), sg1 = ld_g(sg.k0 + 1), su1 = ld_u(sg.k0 + 1);
      if (gu) {
        for (int u = sg.k0; u < sg.k1; ++u) {
          const float sg2 = ld_g(u + 2), su2 = ld_u(u + 2);
          take(v, w2, true);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            a[r] = fmaf(sg0, __uint_as_float(v[r]) + __uint_as_float(v[8 + r]), a[r]);
            b[r] = fmaf(su0, __uint_as_float(w2[r]) + __uint_as_float(w2[8 + r]), b[r]);
          }
          sg0 = sg1;
          su0 = su1;
          sg1 = sg2;
          su1 = su2;
        }
#pragma unroll
        for (int r = 0; r < 8; ++r) {   // n's row scale, a power of two
          a[r] *= c->nsc[r];
          b[r] *= c->nsc[r];
        }
      } else {
        // this expert's activation scales were published with its block
        // counts: acquire them once (the issuer has seen them complete)
        if (tid == 0 && ok) ok = wait_count(p, c, &p.xready[sg.x], (uint32_t)geo.nbi, 4u);
        bar_sync(kBarEpi, 4 * 32);
        const float4* asc =
            reinterpret_cast<const float4*>(p.actb + (size_t)sg.x * f8_act_stride(I, false) + (size_t)I * 16);
        auto ld_a = [&](int u, float4& lo4, float4& hi4) {
          const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
          lo4 = u < sg.k1 ? __ldcg(asc + 2 * u) : z;
          hi4 = u < sg.k1 ? __ldcg(asc + 2 * u + 1) : z;
        };
        // two units per round: one wait and one tensor-memory load latency
        // for the pair (a down stage holds two units); the sums stay in unit
        // order.  The scales of the next pair are loaded before this pair's
        // tiles are waited for.
        float4 al[2], ah[2], nl[2], nh[2];
        float ws[2], nws[2];
        ld_a(sg.k0, al[0], ah[0]);
        ld_a(sg.k0 + 1, al[1], ah[1]);
        ws[0] = ld_g(sg.k0);
        ws[1] = ld_g(sg.k0 + 1);
        for (int u = sg.k0; u < sg.k1; u += 2) {
          const bool two = u + 1 < sg.k1;
          ld_a(u + 2, nl[0], nh[0]);
          ld_a(u + 3, nl[1], nh[1]);
          nws[0] = ld_g(u + 2);
          nws[1] = ld_g(u + 3);
          const uint32_t b0 = t % kF8Acc, b1 = (t + 1) % kF8Acc;
          if (ok) ok = wait_bar(p, c, &c->accfull[b0], (t / kF8Acc) & 1u);
          if (ok && two) ok = wait_bar(p, c, &c->accfull[b1], ((t + 1) / kF8Acc) & 1u);
          tc_fence_after();
          const uint32_t ta = tmem + ((uint32_t)(warp * 32) << 16);
          tmem_ld16_nowait(ta + 32u * b0, v);
          if (two) tmem_ld16_nowait(ta + 32u * b1, w2);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&c->accempty[b0]);
            if (two) mbar_arrive(&c->accempty[b1]);
          }
          t += two ? 2u : 1u;
          const float k0[8] = {al[0].x, al[0].y, al[0].z, al[0].w, ah[0].x, ah[0].y, ah[0].z, ah[0].w};
#pragma unroll
          for (int r = 0; r < 8; ++r) a[r] = fmaf(ws[0] * k0[r], __uint_as_float(v[r]) + __uint_as_float(v[8 + r]), a[r]);
          if (two) {
            const float k1[8] = {al[1].x, al[1].y, al[1].z, al[1].w, ah[1].x, ah[1].y, ah[1].z, ah[1].w};
#pragma unroll
            for (int r = 0; r < 8; ++r)
              a[r] = fmaf(ws[1] * k1[r], __uint_as_float(w2[r]) + __uint_as_float(w2[8 + r]), a[r]);
          }
          al[0] = nl[0];
          ah[0] = nh[0];
          al[1] = nl[1];
          ah[1] = nh[1];
          ws[0] = nws[0];
          ws[1] = nws[1];
        }
      }
      trace(p, 20, t == 1 && tid == 0);
      const bool live = ok && !c->dead;
      if (!epi_combine(p, c, geo, sg, upb, gu, live, i, a, b)) return;
      if (gu) f8_store_act(p, c, sg, live, i, a, b, false);
      else epi_store(p, c, geo, sg, false, live, i, a, b);
    };
    tc_segments(p, geo, L_SGU, 0, seg);
    trace(p, 6, tid == 0);
    if (split) {
      agree();
      bar_sync(kBarEpi, 4 * 32);
      nu = c->nu_comp;
    }
    tc_segments(p, geo, L_RGU, nu, seg);
    trace(p, 7, tid == 0);
    tc_segments(p, geo, L_DN, nu, seg);
    trace(p, 9, tid == 0);
    bar_sync(kBarEpi, 4 * 32);
    if (tid == 0 && may_publish(p, c->epoch, 6, 9)) {
      red_release_add(&p.sync->cnt_y, 1u);
    }
    tc_fence_before();
    bar_arrive(kBarEnd, 5 * 32);   // the issuer may free the tensor memory
  }
  // warps 4-7 have no part in the main phase

  // ==================================================================== tail
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) wait_count(p, c, &p.sync->cnt_y, ep1, 6u);
  bar_sync(kBarCons, kCW * 32);
  tail(p, c, [&](int r, int h) {
    const float* src = p.yp + (size_t)r * (K + 1) * H + h;
    float v[kMaxK + 1];
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j) v[j] = j <= K ? __ldcg(src + (size_t)j * H) : 0.f;
    float y = 0.f;
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j) y += v[j];   // slot order; the zero padding adds exactly
    return y;
  });
  bar_sync(kBarCons, kCW * 32);
  trace(p, 10, tid == 0);
  finish_step(p, c, ep1);
}

}  // namespace mono
