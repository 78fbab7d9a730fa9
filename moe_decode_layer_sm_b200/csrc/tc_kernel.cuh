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
// range the blocks are whole, only the first and last may be partial; the
// CTA that completes a split block last (an atomic per block) adds the parts
// in CTA order, so results do not depend on timing.
//
//   producer (warp 8)   TMA bulk copies into the ring, plus L2 prefetch ahead
//   issuer (warp 9)     one thread: tcgen05.mma A from the ring, B from
//                       shared memory (n for gate/up, activations for down),
//                       D in tensor memory; tcgen05.commit releases slots
//   epilogue (0-3)      tcgen05.ld (warp w: TMEM lanes 32w..32w+31 = rows),
//                       partial tiles, SwiGLU -> activations, down -> yp
//   builders (4-7)      the down B operand: each token row's fp32 activation
//                       as bf16 hi + lo rows (hi = bf16(a), lo = bf16(a - hi))
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
constexpr int kPrefetch = 8;     // stages fetched into L2 ahead of the TMA copy
enum TcList { L_SGU = 0, L_RGU = 1, L_DN = 2 };

// One segment of a CTA's unit range: list, expert entry x (0 = shared),
// block within the expert, units [k0, k1) of the block, the block's global
// index in the list, and the list's unit count.
struct Seg {
  int list, x, blk, k0, k1;
  long long gblk, N;
};

__device__ __forceinline__ long long part_start(long long N, int G, int c) { return (long long)c * N / G; }

// the CTA whose range holds unit u
__device__ __forceinline__ int part_owner(long long N, int G, long long u) {
  int c = (int)((u * G) / N);
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

// Walk this CTA's segments of one list; f(const Seg&).
template <class F>
__device__ __forceinline__ void tc_segments(const Params& p, const TcGeo& g, int list, int nu, F f) {
  const int upb = list == L_DN ? g.upb_dn : g.upb_gu;
  const int nb = list == L_DN ? g.nbh : g.nbi;
  const long long nexp = list == L_SGU ? 1 : list == L_RGU ? nu : nu + 1;
  const long long N = nexp * nb * upb;
  long long a = part_start(N, p.G, blockIdx.x), b = part_start(N, p.G, blockIdx.x + 1);
  while (a < b) {
    const long long gb = a / upb;
    const int k0 = (int)(a % upb);
    const int k1 = (int)min((long long)upb, k0 + (b - a));
    Seg s;
    s.list = list;
    s.x = list == L_SGU ? 0 : list == L_RGU ? (int)(gb / nb) + 1 : (int)(gb / nb);
    s.blk = (int)(gb % nb);
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

  if (tid == 0) {
    c->dead = 0;
    c->lists_ready = 0;
    c->nu = 0;
    c->n_ready = 0;
    c->bld_seq = 0;
    c->mma_seq = 0;
    c->epoch = ld_relaxed(&p.sync->epoch);
    if (ld_relaxed(&p.err->abort)) c->dead = 1;   // fail-stop after an unreported error
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c->accfull[b], 1);
      mbar_init(&c->accempty[b], 4);
    }
    mbar_init(&c->drain, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (c->dead) return;
  if (warp == kMmaWarp) tmem_alloc(&c->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t ep1 = c->epoch + 1u;
  const uint32_t tmem = c->tmem_base;
  trace(p, 0, tid == 0);

  // ================================================================ producer
  if (warp == kProdWarp) {
    uint32_t s = 0, issued = 0;
    bool ok = true;
    auto seg = [&](const Seg& sg) {
      if (lane != 0) return;
      size_t kgb;
      const uint8_t* base = seg_base(p, c, geo, sg, kgb);
      const int kgs = sg.list != L_DN ? kGuKgStage : kDnKgStage;
      const int kg0 = sg.k0 * kKS, kg1 = sg.k1 * kKS;
      const uint32_t bytes = (uint32_t)(kgs * kgb);
      for (int kg = kg0; kg < kg1; kg += kgs) {
        const uint32_t slot = s % p.nst, q = s / p.nst;
        if (ok) {
          const int pk = kg + kPrefetch * kgs;
          if (pk < kg1) prefetch_l2(base + (size_t)pk * kgb, bytes);
          if (q > 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
          if (ok) {
            mbar_arrive_expect_tx(&full[slot], bytes);
            tma_load_1d(ring + (size_t)slot * p.slot_bytes, base + (size_t)kg * kgb, bytes, &full[slot]);
            issued = s + 1;
          }
        }
        ++s;
      }
    };
    // the first stages of each segment go to L2 before its copies start
    auto warm = [&](const Seg& sg) {
      if (lane != 0 || !ok) return;
      size_t kgb;
      const uint8_t* base = seg_base(p, c, geo, sg, kgb);
      const int kgs = sg.list != L_DN ? kGuKgStage : kDnKgStage;
      const int kg0 = sg.k0 * kKS, kg1 = sg.k1 * kKS;
      for (int j = 0; j < kPrefetch && kg0 + j * kgs < kg1; ++j)
        prefetch_l2(base + (size_t)(kg0 + j * kgs) * kgb, (uint32_t)(kgs * kgb));
    };
    tc_segments(p, geo, L_SGU, 0, warm);
    tc_segments(p, geo, L_SGU, 0, seg);
    if (ok && lane == 0) ok = wait_flag(p, c, &c->lists_ready);
    ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    const int nu = ok ? *(volatile int*)&c->nu : 0;
    trace(p, 11, lane == 0);
    tc_segments(p, geo, L_RGU, nu, warm);
    tc_segments(p, geo, L_RGU, nu, seg);
    tc_segments(p, geo, L_DN, nu, warm);
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
    int dgroup = -1;
    if (lane == 0) {
      uint32_t s = 0, t = 0;
      int prev_x = -1;
      bool ok = wait_flag(p, c, &c->n_ready);
      const uint32_t b_addr = smem_u32(regA);
      const uint32_t idesc = umma_idesc_bf16(128, 16);
      auto seg = [&](const Seg& sg) {
        const bool gu = sg.list != L_DN;
        if (!gu && sg.x != prev_x) {
          // a new down expert: hand the previous B operand back once its
          // MMAs are done, then wait for this expert's operand
          if (dgroup >= 0) {
            umma_commit(&c->drain);
            if (ok) ok = wait_bar(p, c, &c->drain, (uint32_t)dgroup & 1u);
            tc_fence_after();
            *(volatile int*)&c->mma_seq = dgroup + 1;
          }
          ++dgroup;
          prev_x = sg.x;
          volatile int* seq = &c->bld_seq;
          const uint64_t t0 = globaltimer();
          while (ok && *seq <= dgroup) {
            if (c->dead) ok = false;
            else if (globaltimer() - t0 > 2 * p.timeout_ns) {
              record_error(p, c, 7u, 4u);
              ok = false;
            }
            __nanosleep(32);
          }
          tc_fence_after();
        }
        const uint32_t buf = t & 1u;
        if (t >= 2 && ok) ok = wait_bar(p, c, &c->accempty[buf], ((t >> 1) - 1) & 1u);
        tc_fence_after();
        const uint32_t d0 = tmem + 32u * buf;
        const int kgs = gu ? kGuKgStage : kDnKgStage;
        const uint32_t kgb = gu ? 4096u : 2048u;
        const int kg0 = sg.k0 * kKS, kg1 = sg.k1 * kKS;
        for (int kg = kg0; kg < kg1; kg += kgs) {
          const uint32_t slot = s % p.nst, q = s / p.nst;
          if (ok) ok = wait_bar(p, c, &full[slot], q & 1);
          tc_fence_after();
          if (ok) {
            const uint32_t a0 = smem_u32(ring + (size_t)slot * p.slot_bytes);
            for (int ks = 0; ks < kgs / 2; ++ks) {
              const uint32_t acc = (kg > kg0 || ks > 0) ? 1u : 0u;
              const uint32_t aa = a0 + (uint32_t)(2 * ks) * kgb;
              const int kb = kg + 2 * ks;   // contraction group of the B operand
              if (gu) {
                const uint64_t db = umma_desc(b_addr + (uint32_t)kb * 128u, 128u, 0u);
                umma_bf16(d0, umma_desc(aa, kgb, 256u), db, idesc, acc);
                umma_bf16(d0 + 16u, umma_desc(aa + 128u, kgb, 256u), db, idesc, acc);
              } else {
                const uint64_t db = umma_desc(b_addr + (uint32_t)kb * 256u, 256u, 128u);
                umma_bf16(d0, umma_desc(aa, kgb, 128u), db, idesc, acc);
              }
            }
          }
          umma_commit(&empty[slot]);
          ++s;
        }
        umma_commit(&c->accfull[buf]);
        ++t;
      };
      tc_segments(p, geo, L_SGU, 0, seg);
      if (ok) ok = wait_flag(p, c, &c->lists_ready);
      const int nu = ok ? *(volatile int*)&c->nu : 0;
      tc_segments(p, geo, L_RGU, nu, seg);
      tc_segments(p, geo, L_DN, nu, seg);
      // every MMA of this CTA is complete before the tensor memory goes away
      umma_commit(&c->drain);
      const uint64_t t0 = globaltimer();
      const uint32_t par = (uint32_t)(dgroup > 0 ? dgroup : 0) & 1u;   // one commit per handed-back operand
      while (!mbar_test(&c->drain, par) && globaltimer() - t0 < p.timeout_ns) __nanosleep(64);
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
    control_warps(p, c, ep1);
    return;
  }
  collapse_norm<true>(p, c, regA);
  fence_proxy_async_smem();   // n is read by the tensor cores (async proxy)
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) *(volatile int*)&c->n_ready = 1;
  trace(p, 3, tid == 0);
  router_logits<true>(p, c, regA);

  // the compute warps agree on the expert list once
  if (tid == 0) {
    const bool ok = wait_flag(p, c, &c->lists_ready);
    c->nu_comp = (ok && !c->dead) ? c->nu : 0;
  }
  bar_sync(kBarCons, kCW * 32);
  const int nu = c->nu_comp;

  if (warp < 4) {
    // ============================================================ epilogue
    // thread <-> row i = 32 w + l of the 128-row tile (its TMEM lane)
    const int i = tid;
    uint32_t t = 0;
    bool ok = true;
    volatile int* bcast = &c->bcast;
    auto seg = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      const int upb = gu ? geo.upb_gu : geo.upb_dn;
      const uint32_t buf = t & 1u;
      if (ok) ok = wait_bar(p, c, &c->accfull[buf], (t >> 1) & 1u);
      tc_fence_after();
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
      // a block split across CTAs: publish this part; the CTA that arrives
      // last adds every part in CTA order
      const long long u0 = sg.gblk * upb, u1 = u0 + upb;
      const int c_lo = part_owner(sg.N, G, u0), c_hi = part_owner(sg.N, G, u1 - 1);
      bool complete = c_lo == c_hi;
      // part slots: a CTA's first and last segment of a list (0 / 1), the
      // routed gate/up list after the shared one (2 / 3)
      const int nsl = gu ? 4 : 2, sl0 = sg.list == L_RGU ? 2 : 0;
      if (!complete) {
        const int slot = sl0 + (part_start(sg.N, G, blockIdx.x) >= u0 ? 0 : 1);
        float* mine = (gu ? p.gpart : p.dpart) + (((size_t)blockIdx.x * nsl + slot) * 128 + i) * 16;
        if (live) {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            mine[r] = a[r];
            mine[8 + r] = b[r];
          }
        }
        __threadfence();
        bar_sync(kBarEpi, 4 * 32);
        if (tid == 0) {
          uint32_t* cnt = (gu ? p.gcnt : p.dcnt) + (size_t)sg.x * (gu ? geo.nbi : geo.nbh) + sg.blk;
          int parts = 0;
          for (int cc = c_lo; cc <= c_hi; ++cc) parts += part_start(sg.N, G, cc) != part_start(sg.N, G, cc + 1);
          const uint32_t old = live ? atomicAdd(cnt, 1u) : 0u;
          const bool last = live && old == (uint32_t)(parts - 1);
          if (last) atomicExch(cnt, 0u);   // ready for the next step
          __threadfence();
          *bcast = last ? 1 : 0;
        }
        bar_sync(kBarEpi, 4 * 32);
        complete = *bcast != 0;
        if (complete) {
#pragma unroll
          for (int r = 0; r < 8; ++r) a[r] = b[r] = 0.f;
          for (int cc = c_lo; cc <= c_hi; ++cc) {
            if (part_start(sg.N, G, cc) == part_start(sg.N, G, cc + 1)) continue;   // empty range
            const int sl = sl0 + (part_start(sg.N, G, cc) >= u0 ? 0 : 1);
            const float* src = (gu ? p.gpart : p.dpart) + (((size_t)cc * nsl + sl) * 128 + i) * 16;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
              a[r] += __ldcg(src + r);
              b[r] += __ldcg(src + 8 + r);
            }
          }
        }
        bar_sync(kBarEpi, 4 * 32);   // bcast is reused by the next segment
      }
      if (!complete || !live) return;
      const int x = sg.x;
      if (gu) {
        const int ch = sg.blk * 128 + i;
#pragma unroll
        for (int r = 0; r < kMaxR; ++r) {
          const int sl = x == 0 ? K : c->uslot[x == 0 ? 0 : x - 1][r];
          if (r < R && sl >= 0) {
            float gg = a[r], uu = b[r];
            if (p.round_bf16) {
              gg = round_bf16(gg);
              uu = round_bf16(uu);
            }
            p.act[((size_t)r * (K + 1) + sl) * I + ch] = gg / (1.0f + expf(-gg)) * uu;
          }
        }
      } else {
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
    };
    tc_segments(p, geo, L_SGU, 0, seg);
    trace(p, 6, tid == 0);
    tc_segments(p, geo, L_RGU, nu, seg);
    trace(p, 7, tid == 0);
    bar_sync(kBarEpi, 4 * 32);
    if (tid == 0) {
      __threadfence();
      red_release_add(&p.sync->cnt_act, 1u);
    }
    tc_segments(p, geo, L_DN, nu, seg);
    trace(p, 9, tid == 0);
    bar_sync(kBarEpi, 4 * 32);
    if (tid == 0) {
      __threadfence();
      red_release_add(&p.sync->cnt_y, 1u);
    }
    tc_fence_before();
    bar_arrive(kBarEnd, 5 * 32);   // the issuer may free the tensor memory
  } else {
    // ======================================================= B builders
    const int bt = tid - 4 * 32;   // 0..127
    if (bt == 0) wait_count(p, c, &p.sync->cnt_act, ep1 * (uint32_t)G, 4u);
    bar_sync(kBarBld, 4 * 32);
    trace(p, 8, bt == 0);
    int dgroup = -1, prev_x = -1;
    auto seg = [&](const Seg& sg) {
      if (sg.x == prev_x) return;
      prev_x = sg.x;
      ++dgroup;
      if (dgroup > 0) {   // the previous operand must be released first
        volatile int* seq = &c->mma_seq;
        const uint64_t t0 = globaltimer();
        while (*seq < dgroup && !c->dead) {
          if (globaltimer() - t0 > 2 * p.timeout_ns) {
            record_error(p, c, 7u, 4u);
            break;
          }
          __nanosleep(32);
        }
      }
      const int x = sg.x;
      // layout [kg][2 row groups][8 rows][8]: row 2r = hi, 2r + 1 = lo of
      // token row r; rows of tokens that do not use the expert are zero
      for (int q = bt; q < geo.kgi * 8; q += 128) {
        const int kg = q / 8, r = q % 8;
        int sl = -1;
        if (r < R) sl = x == 0 ? K : c->uslot[x - 1][r];
        uint4 hi = make_uint4(0u, 0u, 0u, 0u), lo = make_uint4(0u, 0u, 0u, 0u);
        if (sl >= 0 && !c->dead) {
          const float4* src = reinterpret_cast<const float4*>(p.act + ((size_t)r * (K + 1) + sl) * I + kg * 8);
          const float4 a = __ldcg(src), b = __ldcg(src + 1);
          const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float h0 = round_bf16(f[2 * k]), h1 = round_bf16(f[2 * k + 1]);
            hw[k] = pack_bf16x2(h0, h1);
            lw[k] = pack_bf16x2(f[2 * k] - h0, f[2 * k + 1] - h1);
          }
          hi = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          lo = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
        uint8_t* blk = regA + (size_t)kg * 256;
        *reinterpret_cast<uint4*>(blk + (size_t)(2 * r) * 16) = hi;
        *reinterpret_cast<uint4*>(blk + (size_t)(2 * r + 1) * 16) = lo;
      }
      fence_proxy_async_smem();
      bar_sync(kBarBld, 4 * 32);
      if (bt == 0) *(volatile int*)&c->bld_seq = dgroup + 1;
    };
    tc_segments(p, geo, L_DN, nu, seg);
  }

  // ==================================================================== tail
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) wait_count(p, c, &p.sync->cnt_y, ep1 * (uint32_t)G, 6u);
  bar_sync(kBarCons, kCW * 32);
  tail(p, c, [&](int r, int h) {
    float y = 0.f;
    const float* src = p.yp + (size_t)r * (K + 1) * H + h;
    for (int j = 0; j <= K; ++j) y += __ldcg(src + (size_t)j * H);
    return y;
  });
  bar_sync(kBarCons, kCW * 32);
  trace(p, 10, tid == 0);
  finish_step(p, c, ep1);
}

}  // namespace mono
