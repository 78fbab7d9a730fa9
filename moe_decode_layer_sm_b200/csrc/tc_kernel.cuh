// Tensor-core variant of the persistent kernel (bf16 experts): the expert
// matvecs run on the 5th-generation tensor cores.
//
// Weights are packed in blocks of 128 output rows (16 rowgroups of 8):
//   gate/up [E+1][I/128][H/8][16 rowgroups][gate | up][8 rows][8] bf16
//   down    [E+1][H/128][I/8][16 rowgroups][8 rows][8] bf16
// so one ring stage (16 KB: 4 contraction groups of gate/up, 8 of down) is
// one contiguous TMA bulk copy, and one tcgen05.mma covers M = 128 rows x
// K = 16 (4 KB of weights).  Work is cut in units of (block, 128 contraction
// elements) and every CTA takes an equal contiguous range of units: inside a
// range the blocks are whole, only the first and last may be partial; one
// CTA adds a split block's parts in CTA order (epi_combine), so results do
// not depend on timing.
//
//   producer (warp 8)   TMA bulk copies into the ring (the ring's depth is
//                       what keeps enough bytes in flight: an L2 prefetch
//                       ahead of it only queues on the same copy engine)
//   issuer (warp 9)     one thread: tcgen05.mma A from the ring, B from
//                       shared memory (n for gate/up, activations for down,
//                       one bulk copy per down expert), D in tensor memory;
//                       tcgen05.commit releases slots
//   epilogue (0-3)      tcgen05.ld (warp w: TMEM lanes 32w..32w+31 = rows),
//                       partial tiles, SwiGLU written straight in the down
//                       B operand's layout: each token row's fp32 activation
//                       as bf16 hi + lo rows (hi = bf16(a), lo = bf16(a - hi));
//                       down -> yp
//
// B operands have N = 16 columns.  Gate/up uses the 8 rows of n twice (the
// descriptor's row-group stride is 0: columns 8-15 repeat 0-7); down uses
// rows 2r (hi) and 2r + 1 (lo) of token row r.
#pragma once
#include "common.cuh"

namespace mono {

constexpr int kTmemCols = 64;    // two accumulator buffers of 32 columns (gate 16 | up 16)
constexpr int kKS = 16;          // contraction groups (of 8) per work unit
constexpr int kGuKgStage = 4;    // contraction groups per ring stage, gate/up (4 KB each)
constexpr int kDnKgStage = 8;    // contraction groups per ring stage, down (2 KB each)
enum TcList { L_SGU = 0, L_RGU = 1, L_DN = 2 };

// One segment of a CTA's unit range: list, expert entry x (0 = shared),
// block within the expert, units [k0, k1) of the block, the block's global
// index in the list, and the list's unit count.
struct Seg {
  int list, x, blk, k0, k1;
  long long gblk, N;
};

// 32-bit arithmetic: the plan keeps every list's units times the grid below
// 2^31 (64-bit division is a long software sequence, on the critical path of
// every segment's combine)
__device__ __forceinline__ long long part_start(long long N, int G, int c) {
  return (long long)((uint32_t)c * (uint32_t)N / (uint32_t)G);
}

// the CTA whose range holds unit u
__device__ __forceinline__ int part_owner(long long N, int G, long long u) {
  int c = (int)((uint32_t)u * (uint32_t)G / (uint32_t)N);
  while (c + 1 < G && part_start(N, G, c + 1) <= u) ++c;
  while (c > 0 && part_start(N, G, c) > u) --c;
  return c;
}

struct TcGeo {
  int nbi, nbh, kgh, kgi;   // blocks of I and of H; contraction groups of H and of I
  int upb_gu, upb_dn;       // units per block
  __device__ TcGeo(const Params& p) {
    nbi = p.I / 128;
    nbh = p.H / 128;
    kgh = p.H / 8;
    kgi = p.I / 8;
    upb_gu = kgh / kKS;
    upb_dn = kgi / kKS;
  }
};

// The shared gate/up list is cut along its blocks: block b goes to CTAs
// [sgu_c0(b), sgu_c0(b + 1)), which split its units evenly, so that no CTA
// holds parts of two blocks.  (A CTA that holds a block's end and the next
// block's start finishes two blocks; the second one then completes while
// the routed weights saturate HBM, where every round trip of its combine
// takes microseconds, and stalls that CTA's MMAs.)  Used when every block
// has a CTA of its own.
__device__ __forceinline__ bool sgu_by_block(const Params& p, const TcGeo& g) { return p.G >= g.nbi; }
__device__ __forceinline__ int sgu_c0(const Params& p, const TcGeo& g, int b) { return (b * p.G + g.nbi - 1) / g.nbi; }
// units [k0, k1) of block b for the j-th of its m CTAs
__device__ __forceinline__ void sgu_share(const TcGeo& g, int j, int m, int& k0, int& k1) {
  k0 = j * g.upb_gu / m;
  k1 = (j + 1) * g.upb_gu / m;
}

// Walk this CTA's segments of one list; f(const Seg&).
template <class F>
__device__ __forceinline__ void tc_segments(const Params& p, const TcGeo& g, int list, int nu, F f) {
  if (list == L_SGU && sgu_by_block(p, g)) {
    const int b = (int)(((long long)blockIdx.x * g.nbi) / p.G);
    const int c0 = sgu_c0(p, g, b), m = sgu_c0(p, g, b + 1) - c0;
    Seg s;
    sgu_share(g, (int)blockIdx.x - c0, m, s.k0, s.k1);
    if (s.k0 < s.k1) {
      s.list = L_SGU;
      s.x = 0;
      s.blk = b;
      s.gblk = b;
      s.N = (long long)g.nbi * g.upb_gu;
      f(s);
    }
    return;
  }
  const int upb = list == L_DN ? g.upb_dn : g.upb_gu;
  const int nb = list == L_DN ? g.nbh : g.nbi;
  const long long nexp = list == L_SGU ? 1 : list == L_RGU ? nu : nu + 1;
  const long long N = nexp * nb * upb;
  long long a = part_start(N, p.G, blockIdx.x), b = part_start(N, p.G, blockIdx.x + 1);
  while (a < b) {
    const long long gb = (uint32_t)a / (uint32_t)upb;
    const int k0 = (int)((uint32_t)a % (uint32_t)upb);
    const int k1 = (int)min((long long)upb, k0 + (b - a));
    Seg s;
    s.list = list;
    s.x = list == L_SGU ? 0 : list == L_RGU ? (int)((uint32_t)gb / (uint32_t)nb) + 1 : (int)((uint32_t)gb / (uint32_t)nb);
    s.blk = (int)((uint32_t)gb % (uint32_t)nb);
    s.k0 = k0;
    s.k1 = k1;
    s.gblk = gb;
    s.N = N;
    f(s);
    a += k1 - k0;
  }
}

__device__ __forceinline__ int seg_expert(const Params& p, const Ctl* c, int x) { return x == 0 ? p.E : c->ulist[x - 1]; }

// first byte of a segment's block and the bytes of one contraction group of it
__device__ __forceinline__ const uint8_t* seg_base(const Params& p, const Ctl* c, const TcGeo& g, const Seg& sg,
                                                   size_t& kgb) {
  const int e = seg_expert(p, c, sg.x);
  if (sg.list != L_DN) {
    kgb = 4096;
    return p.gu + (size_t)e * p.gu_estride + (size_t)sg.blk * g.kgh * kgb;
  }
  kgb = 2048;
  return p.dn + (size_t)e * p.dn_estride + (size_t)sg.blk * g.kgi * kgb;
}

// Epilogue, thread i (= row i of the 128-row tile) of warps 0-3, with this
// CTA's part of a block in a[8] (gate, or the down output) and b[8] (up):
// for a split block, publish the part; one CTA (the lowest holder, or on the
// shared list the last to arrive) adds the parts in CTA order.  A part is
// [a0..a7 | b0..b7] of this row, only the quarters in use.  Returns true in the
// CTA that holds the complete block (then a and b hold its sums); the same
// answer in every epilogue thread.
__device__ __forceinline__ bool epi_combine(const Params& p, Ctl* c, const TcGeo& geo, const Seg& sg, int upb, bool gu,
                                            bool live, int i, float (&a)[8], float (&b)[8]) {
  const int G = p.G, R = p.R, tid = threadIdx.x;
  volatile int* bcast = &c->bcast;
  const long long u0 = sg.gblk * upb, u1 = u0 + upb;
  const bool by_block = sg.list == L_SGU && sgu_by_block(p, geo);   // one segment per CTA, slot 0
  const int c_lo = by_block ? sgu_c0(p, geo, sg.blk) : part_owner(sg.N, G, u0);
  const int c_hi = by_block ? sgu_c0(p, geo, sg.blk + 1) - 1 : part_owner(sg.N, G, u1 - 1);
  // does CTA cc hold a part of this block, and in which slot
  auto holds = [&](int cc) {
    if (!by_block) return part_start(sg.N, G, cc) != part_start(sg.N, G, cc + 1);
    int k0, k1;
    sgu_share(geo, cc - c_lo, c_hi - c_lo + 1, k0, k1);
    return k0 < k1;
  };
  auto slot_of = [&](int cc, int sl0) { return by_block ? 0 : sl0 + (part_start(sg.N, G, cc) >= u0 ? 0 : 1); };
  if (c_lo == c_hi) return true;
  // part slots: a CTA's first and last segment of a list (0 / 1), the
  // routed gate/up list after the shared one (2 / 3)
  const int nsl = gu ? 4 : 2, sl0 = sg.list == L_RGU ? 2 : 0;
  const bool q1 = R > 4;
  const int slot = slot_of((int)blockIdx.x, sl0);
  float4* mine = reinterpret_cast<float4*>((gu ? p.gpart : p.dpart) + (((size_t)blockIdx.x * nsl + slot) * 128 + i) * 16);
  if (!by_block) {
    // A list cut in contiguous ranges: the block runs past c_lo's range, so
    // c_lo's part is its last segment of the list, computed after every
    // other holder's (each one's first segment, or its whole range).  c_lo
    // adds the parts; the others publish theirs and go on.
    uint32_t* cnt = (gu ? p.gcnt : p.dcnt) + (size_t)sg.x * (gu ? geo.nbi : geo.nbh) + sg.blk;
    if ((int)blockIdx.x != c_lo) {
      if (live) {
        __stcg(mine, make_float4(a[0], a[1], a[2], a[3]));
        if (q1) __stcg(mine + 1, make_float4(a[4], a[5], a[6], a[7]));
        if (gu) __stcg(mine + 2, make_float4(b[0], b[1], b[2], b[3]));
        if (gu && q1) __stcg(mine + 3, make_float4(b[4], b[5], b[6], b[7]));
      }
      bar_sync(kBarEpi, 4 * 32);
      if (tid == 0 && live && may_publish(p, c->epoch, 0, 5 + (uint32_t)sg.list)) red_release_add(cnt, 1u);
      return false;
    }
    if (tid == 0 && live) {
      int parts = 0;
      for (int cc = c_lo; cc <= c_hi; ++cc) parts += holds(cc) ? 1 : 0;
      if (wait_count(p, c, cnt, (uint32_t)(parts - 1), gu ? 4u : 6u)) *cnt = 0u;   // ready for the next step
    }
    bar_sync(kBarEpi, 4 * 32);
    // this CTA's own part first (it is c_lo), then the others in CTA order,
    // four in flight at a time: the additions of the general path below
    for (int cb = c_lo + 1; cb <= c_hi; cb += 4) {
      float4 ld[4][4];
      bool use[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = cb + j;
        use[j] = live && cc <= c_hi && holds(cc);
        const float4* src =
            reinterpret_cast<const float4*>((gu ? p.gpart : p.dpart) + (((size_t)cc * nsl + slot_of(cc, sl0)) * 128 + i) * 16);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        ld[j][0] = use[j] ? __ldcg(src) : z;
        ld[j][1] = use[j] && q1 ? __ldcg(src + 1) : z;
        ld[j][2] = use[j] && gu ? __ldcg(src + 2) : z;
        ld[j][3] = use[j] && gu && q1 ? __ldcg(src + 3) : z;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!use[j]) continue;
        a[0] += ld[j][0].x; a[1] += ld[j][0].y; a[2] += ld[j][0].z; a[3] += ld[j][0].w;
        a[4] += ld[j][1].x; a[5] += ld[j][1].y; a[6] += ld[j][1].z; a[7] += ld[j][1].w;
        b[0] += ld[j][2].x; b[1] += ld[j][2].y; b[2] += ld[j][2].z; b[3] += ld[j][2].w;
        b[4] += ld[j][3].x; b[5] += ld[j][3].y; b[6] += ld[j][3].z; b[7] += ld[j][3].w;
      }
    }
    if (!q1) {
#pragma unroll
      for (int r = 4; r < 8; ++r) a[r] = b[r] = 0.f;   // the general path adds zeros there
    }
    if (!gu) {
#pragma unroll
      for (int r = 0; r < 8; ++r) b[r] = 0.f;
    }
    return true;
  }
  if (live) {
    __stcg(mine, make_float4(a[0], a[1], a[2], a[3]));
    if (q1) __stcg(mine + 1, make_float4(a[4], a[5], a[6], a[7]));
    if (gu) __stcg(mine + 2, make_float4(b[0], b[1], b[2], b[3]));
    if (gu && q1) __stcg(mine + 3, make_float4(b[4], b[5], b[6], b[7]));
  }
  __threadfence();
  bar_sync(kBarEpi, 4 * 32);
  if (tid == 0) {
    uint32_t* cnt = (gu ? p.gcnt : p.dcnt) + (size_t)sg.x * (gu ? geo.nbi : geo.nbh) + sg.blk;
    int parts = 0;
    for (int cc = c_lo; cc <= c_hi; ++cc) parts += holds(cc) ? 1 : 0;
    if (live) may_publish(p, c->epoch, 0, 5 + (uint32_t)sg.list);
    const uint32_t old = live ? atomicAdd(cnt, 1u) : 0u;
    const bool last = live && old == (uint32_t)(parts - 1);
    if (last) atomicExch(cnt, 0u);   // ready for the next step
    __threadfence();
    *bcast = last ? 1 : 0;
  }
  bar_sync(kBarEpi, 4 * 32);
  const bool complete = *bcast != 0;
  if (complete) {
#pragma unroll
    for (int r = 0; r < 8; ++r) a[r] = b[r] = 0.f;
    // four parts in flight at a time, added in CTA order
    for (int cb = c_lo; cb <= c_hi; cb += 4) {
      float4 ld[4][4];
      bool use[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int cc = cb + j;
        use[j] = cc <= c_hi && holds(cc);   // skip empty ranges
        const int sl = slot_of(cc, sl0);
        const float4* src =
            reinterpret_cast<const float4*>((gu ? p.gpart : p.dpart) + (((size_t)cc * nsl + sl) * 128 + i) * 16);
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        ld[j][0] = use[j] ? __ldcg(src) : z;
        ld[j][1] = use[j] && q1 ? __ldcg(src + 1) : z;
        ld[j][2] = use[j] && gu ? __ldcg(src + 2) : z;
        ld[j][3] = use[j] && gu && q1 ? __ldcg(src + 3) : z;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (!use[j]) continue;
        a[0] += ld[j][0].x; a[1] += ld[j][0].y; a[2] += ld[j][0].z; a[3] += ld[j][0].w;
        a[4] += ld[j][1].x; a[5] += ld[j][1].y; a[6] += ld[j][1].z; a[7] += ld[j][1].w;
        b[0] += ld[j][2].x; b[1] += ld[j][2].y; b[2] += ld[j][2].z; b[3] += ld[j][2].w;
        b[4] += ld[j][3].x; b[5] += ld[j][3].y; b[6] += ld[j][3].z; b[7] += ld[j][3].w;
      }
    }
  }
  bar_sync(kBarEpi, 4 * 32);   // bcast is reused by the next segment
  return complete;
}

// A complete block.  Gate/up: SwiGLU, written as the down projection's B
// operand of expert entry x, [I/8][16 rows][8] 16-bit, row 2r = hi, 2r + 1 =
// lo of token row r (bf16), zero for rows that do not
// use the expert; then the block counts for its expert.  Down: the weighted
// output of every row that uses the expert into yp.
__device__ __forceinline__ void epi_store(const Params& p, Ctl* c, const TcGeo& geo, const Seg& sg, bool gu, bool live,
                                          int i, const float (&a)[8], const float (&b)[8]) {
  const int R = p.R, K = p.K, H = p.H, I = p.I, tid = threadIdx.x;
  const int x = sg.x;
  if (gu) {
    const int ch = sg.blk * 128 + i;
    uint16_t* dst = reinterpret_cast<uint16_t*>(p.actb + (size_t)x * I * 32 + (size_t)(ch >> 3) * 256) + (ch & 7);
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) {
      if (!live) break;
      const int sl = x == 0 ? K : c->uslot[x == 0 ? 0 : x - 1][r];
      uint16_t hb = 0, lb = 0;
      if (r < R && sl >= 0) {
        float gg = a[r], uu = b[r];
        if (p.round_bf16) {
          gg = round_bf16(gg);
          uu = round_bf16(uu);
        }
        const float act = gg / (1.0f + expf(-gg)) * uu;
        const __nv_bfloat16 hi = __float2bfloat16_rn(act);
        hb = __bfloat16_as_ushort(hi);
        lb = __bfloat16_as_ushort(__float2bfloat16_rn(act - __bfloat162float(hi)));
      }
      dst[(2 * r) * 8] = hb;
      dst[(2 * r + 1) * 8] = lb;
    }
    // the block's activations are out: count it for its expert (they are
    // read by bulk copies, the async proxy)
    __threadfence();
    bar_sync(kBarEpi, 4 * 32);   // reached by every epilogue thread, live or not
    // (fault injection at the activation stage: the arrival of the shared
    // expert's first block is withheld, whichever CTA completes it)
    if (tid == 0 && live && may_publish(p, c->epoch, 0, 8) && !(p.fault_stage == 4 && x == 0 && sg.blk == 0)) {
      fence_proxy_async_global();
      red_release_add(&p.xready[x], 1u);
    }
  } else if (live) {
    const int h = sg.blk * 128 + i;
#pragma unroll
    for (int r = 0; r < kMaxR; ++r) {
      const int sl = x == 0 ? K : c->uslot[x == 0 ? 0 : x - 1][r];
      if (r < R && sl >= 0) {
        const float wgt = x == 0 ? 1.0f : c->wt[r][sl];
        p.yp[((size_t)r * (K + 1) + sl) * H + h] = wgt * a[r];
      }
    }
  }
}

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) mono_ffn_tc_kernel(const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  const SmemLayout L(p.nst, p.slot_bytes, p.regA_bytes, p.ymax);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + p.nst;
  Ctl* c = reinterpret_cast<Ctl*>(smem + L.ctl);
  uint8_t* regA = smem + L.regA;   // n (gate/up B operand), then the down B operand
  uint8_t* ring = smem + L.ring;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int R = p.R, H = p.H, I = p.I, K = p.K, G = p.G;
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
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
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
  if (warp == kMmaWarp) tmem_alloc(&c->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t ep1 = c->epoch + (uint32_t)G;   // every grid counter's target in this launch
  const uint32_t tmem = c->tmem_base;
  trace(p, 0, tid == 0);
  if (p.trace && tid == 0) {   // which SM this CTA runs on
    uint32_t sm;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(sm));
    p.trace[blockIdx.x * kTracePoints + 31] = sm;
  }

  // ================================================================ producer
  if (warp == kProdWarp) {
    uint32_t s = 0, issued = 0;
    bool ok = true;
    uint32_t first_copy = 0u;
    bool dry = false;
    auto seg = [&](const Seg& sg) {
      if (lane != 0) return;
      size_t kgb;
      const uint8_t* base = seg_base(p, c, geo, sg, kgb);
      const int kgs = sg.list != L_DN ? kGuKgStage : kDnKgStage;
      const int kg0 = sg.k0 * kKS, kg1 = sg.k1 * kKS;
      const uint32_t bytes = (uint32_t)(kgs * kgb);
      for (int kg = kg0; kg < kg1; kg += kgs) {
        const uint32_t slot = s % p.nst, q = s / p.nst;
        if (ok && !dry) {
          if (q > 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
          if (ok) {
            mbar_arrive_expect_tx(&full[slot], bytes);
            tma_load_1d(ring + (size_t)slot * p.slot_bytes, base + (size_t)kg * kgb, bytes, &full[slot]);
            issued = s + 1;
            if (sg.list != L_SGU && !(first_copy & (1u << sg.list))) {
              first_copy |= 1u << sg.list;
              trace(p, 17 + sg.list);
            }
          }
        }
        ++s;
      }
    };
    if (lane == 0) {
      // the prologue's later inputs go to L2 ahead of the weight stream:
      // this CTA's router rows, the norm weights and the router bias
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
  // The whole warp runs the loop (waits in lane 0, results broadcast), one
  // elected lane issues the MMAs and commits.
  if (warp == kMmaWarp) {
    uint32_t s = 0, t = 0, ndrain = 0, nb = 0;
    int prev_x = -1;
    bool first_rgu = true, b_pending = false;
    auto warp_ok = [&](bool v) { return __shfl_sync(0xffffffffu, (int)v, 0) != 0; };
    bool ok = true;
    if (lane == 0) ok = wait_flag(p, c, &c->n_ready);
    ok = warp_ok(ok);
    const uint32_t b_addr = smem_u32(regA);
    const uint32_t idesc = umma_idesc_bf16(128, 16);
    const uint32_t b_bytes = (uint32_t)I * 32u;
    // descriptors: the start address sits in the low 14 bits (in 16-byte
    // units), so moving an operand by d bytes adds d >> 4
    const uint64_t bdesc_gu = umma_desc(b_addr, 128u, 0u), bdesc_dn = umma_desc(b_addr, 256u, 128u);
    auto seg = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      if (!gu && sg.x != prev_x) {
        // a new down expert: once every MMA reading the B region is done
        // (and, the first time, every CTA's activations are out), one bulk
        // copy brings this expert's operand in
        // this expert's activations are complete once every one of its
        // gate/up blocks has been finished (by whichever CTA)
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
            tma_load_1d(regA, p.actb + (size_t)sg.x * b_bytes, b_bytes, &c->bfull);
            ok = wait_bar(p, c, &c->bfull, nb & 1u);
          }
          ok = warp_ok(ok);
          b_pending = !ok;
          ++nb;
        }
        tc_fence_after();
        trace(p, 15, nb == 1 && lane == 0);
      }
      const uint32_t buf = t & 1u;
      if (t >= 2) {
        if (lane == 0 && ok) ok = wait_bar(p, c, &c->accempty[buf], ((t >> 1) - 1) & 1u);
        ok = warp_ok(ok);
      }
      tc_fence_after();
      const uint32_t d0 = tmem + 32u * buf;
      const int kgs = gu ? kGuKgStage : kDnKgStage;
      const uint32_t kgb = gu ? 4096u : 2048u;
      const int kg0 = sg.k0 * kKS, kg1 = sg.k1 * kKS;
      for (int kg = kg0; kg < kg1; kg += kgs) {
        const uint32_t slot = s % p.nst, q = s / p.nst;
        if (lane == 0 && ok) ok = wait_bar(p, c, &full[slot], q & 1);
        ok = warp_ok(ok);
        tc_fence_after();
        if (sg.list == L_RGU && first_rgu) {
          first_rgu = false;
          trace(p, 13, lane == 0);
        }
        if (ok) {
          const uint64_t adesc = umma_desc(smem_u32(ring + (size_t)slot * p.slot_bytes), kgb, gu ? 256u : 128u);
          if (gu) {
            const uint64_t bd = bdesc_gu + (uint64_t)(kg * 8);   // kg * 128 bytes
#pragma unroll
            for (int ks = 0; ks < kGuKgStage / 2; ++ks) {
              const uint32_t acc = (kg > kg0 || ks > 0) ? 1u : 0u;
              const uint64_t da = adesc + (uint64_t)(ks * 512);   // 2 ks * 4096 bytes
              const uint64_t db = bd + (uint64_t)(ks * 16);        // 2 ks * 128 bytes
              umma_bf16_warp(d0, da, db, idesc, acc);
              umma_bf16_warp(d0 + 16u, da + 8u, db, idesc, acc);   // up: 128 bytes on
            }
          } else {
            const uint64_t bd = bdesc_dn + (uint64_t)(kg * 16);  // kg * 256 bytes
#pragma unroll
            for (int ks = 0; ks < kDnKgStage / 2; ++ks) {
              const uint32_t acc = (kg > kg0 || ks > 0) ? 1u : 0u;
              umma_bf16_warp(d0, adesc + (uint64_t)(ks * 256), bd + (uint64_t)(ks * 32), idesc, acc);
            }
          }
        }
        umma_commit_warp(&empty[slot]);
        ++s;
      }
      umma_commit_warp(&c->accfull[buf]);
      ++t;
    };
    tc_segments(p, geo, L_SGU, 0, seg);
    if (lane == 0 && ok) ok = wait_flag(p, c, &c->lists_ready);
    ok = warp_ok(ok);
    const int nu = ok ? *(volatile int*)&c->nu : 0;
    tc_segments(p, geo, L_RGU, nu, seg);
    trace(p, 14, lane == 0);
    tc_segments(p, geo, L_DN, nu, seg);
    trace(p, 16, lane == 0);
    // every MMA of this CTA is complete before the tensor memory goes
    // away, and no bulk copy still targets shared memory at exit
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
    tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // ================================================================ prologue
  prologue_mix(p, c, regA, ep1);
  if (warp >= kCtlWarp0) {
    control_warps(p, c, regA, ep1, false, p.R <= 4);
    return;
  }
  collapse_norm<true>(p, c, regA, ep1);
  fence_proxy_async_smem();   // n is read by the tensor cores (async proxy)
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) *(volatile int*)&c->n_ready = 1;
  trace(p, 3, tid == 0);
  router_logits<true>(p, c, regA, false);
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
    auto seg = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      const int upb = gu ? geo.upb_gu : geo.upb_dn;
      const uint32_t buf = t & 1u;
      if (ok) ok = wait_bar(p, c, &c->accfull[buf], (t >> 1) & 1u);
      tc_fence_after();
      trace(p, 20, t == 0 && tid == 0);
      uint32_t v[16], w2[16];
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + 32u * buf, v);
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + 32u * buf + 16u, w2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c->accempty[buf]);
      ++t;
      const bool live = ok && !c->dead;
      // this tile's value per token row: gate and up, or the down output with
      // its hi and lo columns added
      float a[8], b[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        if (gu) {
          a[r] = __uint_as_float(v[r]);
          b[r] = __uint_as_float(w2[r]);
        } else {
          a[r] = __uint_as_float(v[2 * r]) + __uint_as_float(v[2 * r + 1]);
          b[r] = 0.f;
        }
      }
      if (!epi_combine(p, c, geo, sg, upb, gu, live, i, a, b)) return;
      epi_store(p, c, geo, sg, gu, live, i, a, b);
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
