// Tensor-core variant of the persistent kernel for quantised experts: FP8
// e4m3 with one fp32 scale per 1 x 128 block, and MXFP4 (e2m1 with one e8m0
// scale per 32 elements).  Same work units, lists, split-block combine and
// prologue as the bf16 tensor-core kernel; what differs is the A operand.
//
// The weights stream through the ring as codes.  Warps 4-7 (idle in the
// bf16 kernel's main phase) convert them, one thread per weight row, to fp16
// and write them into tensor memory with tcgen05.st; the MMA reads A from
// tensor memory (M = 128 rows, K = 16, fp16) and B (n, or the activations)
// from shared memory, in fp16.  The conversions are exact: every e4m3 value
// is an fp16 value, and an e2m1 value times its power-of-two MXFP4 scale is
// one as long as the scale lies in [2^-22, 2^12] (the plan checks the packed
// scales).  Only the FP8 block scale is not a power of two: it multiplies
// the fp32 partial product of its 128-element unit in the epilogue, so each
// FP8 unit gets its own accumulator.
//
// Packed units (one unit = 128 weight rows x 128 contraction elements of one
// matrix), 16-byte chunk j of row i at [j][i] so that the 32 converter lanes
// of a warp read consecutive 16-byte words:
//   FP8    codes [8 chunks][128 rows][16]                      16384 B
//   MXFP4  codes [4 chunks][128 rows][16], scales [128 rows][4]  8704 B
// gate/up units hold gate then up; FP8 scales sit in their own arrays
// (read by the epilogue), MXFP4 scales travel with the codes.
#pragma once
#include "tc_kernel.cuh"

namespace mono {

constexpr int kTqTmemCols = 512;   // 2 accumulators of 32 columns, then 3 A buffers of 128
constexpr uint32_t kAbCol = 64;    // first A buffer; buffer b at kAbCol + 128 b (gate 64 | up 64)
constexpr int kAb = kMaxAb;        // A buffers: the converters run up to 3 units ahead of the MMAs
// accumulator buffer b: columns 32 b for b < 2, behind the A buffers for b >= 2
__device__ __forceinline__ uint32_t acc_col(uint32_t b) { return b < 2 ? 32u * b : 448u + 32u * (b - 2); }
static_assert(kTqTmemCols >= (int)kAbCol + 128 * kAb, "A buffers fit in the tensor memory");

template <int WT> struct TqFmt;
template <> struct TqFmt<W_FP8> {
  static constexpr int CHUNKS = 8, CODE_BYTES = 16384, MAT_BYTES = 16384;
};
template <> struct TqFmt<W_FP4> {
  static constexpr int CHUNKS = 4, CODE_BYTES = 8192, MAT_BYTES = 8192 + 512;
};

// fp16 bits of 2^(e - 127) for an e8m0 code e with e - 127 in [-22, 12]
__device__ __forceinline__ uint32_t e8m0_to_h(uint32_t e) {
  const int k = (int)e - 127;
  return k >= -14 ? (uint32_t)(k + 15) << 10 : 1u << (k + 24);
}

// Chunks [j0, j1) of one matrix of one unit from the ring slot to this
// thread's lane (row) of tensor memory, from column taddr on (64 columns
// for the whole matrix).
template <int WT>
__device__ __forceinline__ void tq_convert(const uint8_t* mat, int row, uint32_t taddr, int j0, int j1) {
  using F = TqFmt<WT>;
  if (WT == W_FP8) {
#pragma unroll
    for (int j = 0; j < F::CHUNKS; j += 2) {
      if (j < j0 || j >= j1) continue;
      uint32_t v[16];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 q = *reinterpret_cast<const uint4*>(mat + (size_t)(j + h) * 2048 + row * 16);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          v[8 * h + 2 * m] = e4m3x2_to_h2(w[m] & 0xFFFFu);
          v[8 * h + 2 * m + 1] = e4m3x2_to_h2(w[m] >> 16);
        }
      }
      tmem_st16(taddr + 8u * j, v);
    }
  } else {
    const uint32_t sc = *reinterpret_cast<const uint32_t*>(mat + F::CODE_BYTES + row * 4);
#pragma unroll
    for (int j = 0; j < F::CHUNKS; ++j) {
      if (j < j0 || j >= j1) continue;
      const uint32_t s1 = e8m0_to_h((sc >> (8 * j)) & 0xFFu);
      const uint32_t s2 = s1 | (s1 << 16);
      const uint4 q = *reinterpret_cast<const uint4*>(mat + (size_t)j * 2048 + row * 16);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t v[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) v[m] = hmul2_bits(e2m1x2_to_h2((w[m >> 2] >> (8 * (m & 3))) & 0xFFu), s2);
      tmem_st16(taddr + 16u * j, v);
    }
  }
}

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) mono_ffn_tq_kernel(const __grid_constant__ Params p) {
  using F = TqFmt<WT>;
  constexpr uint32_t MAT = F::MAT_BYTES;
  constexpr bool PER_UNIT = WT == W_FP8;   // a non-power-of-two block scale per unit
  // MXFP4 (two codes a byte, a scale multiply each) needs the conversion
  // throughput of all eight compute warps; its epilogue runs once a segment
  // on warps 0-3 between their conversions.  FP8 converts on warps 4-7.
  constexpr int NCV = WT == W_FP4 ? 8 : 4;
  // FP8 hands every unit to the epilogue: four accumulators keep the MMAs
  // three units ahead of it; MXFP4 hands over once per segment
  constexpr uint32_t NACC = PER_UNIT ? 4 : 2;
  static_assert(NACC <= kMaxAcc && 448 + 32 * 2 <= kTqTmemCols, "accumulators fit");
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
    c->epoch = ld_relaxed(&p.sync->epoch);
    if (ld_relaxed(&p.err->abort)) c->dead = 1;   // fail-stop after an unreported error
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NCV);   // the converter warps
    }
    for (uint32_t b = 0; b < NACC; ++b) {
      mbar_init(&c->accfull[b], 1);
      mbar_init(&c->accempty[b], 4);
    }
    for (int b = 0; b < kAb; ++b) {
      mbar_init(&c->abfull[b], NCV);
      mbar_init(&c->abempty[b], 1);
    }
    mbar_init(&c->drain, 1);
    mbar_init(&c->bfull, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (c->dead) return;
  if (warp == kMmaWarp) tmem_alloc(&c->tmem_base, kTqTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t ep1 = c->epoch + 1u;
  const uint32_t tmem = c->tmem_base;
  trace(p, 0, tid == 0);

  // unit bytes in the ring and the first byte of a segment's block; a ring
  // stage holds one gate/up unit or two down units (one copy of 2 MAT bytes:
  // a single down unit of MXFP4 would be a copy too small to stream well)
  auto unit_bytes = [&](const Seg& sg) { return sg.list != L_DN ? 2u * MAT : MAT; };
  auto stage_units = [&](const Seg& sg) { return sg.list != L_DN ? 1 : 2; };
  auto block_base = [&](const Seg& sg) -> const uint8_t* {
    const int e = seg_expert(p, c, sg.x);
    if (sg.list != L_DN) return p.gu + (size_t)e * p.gu_estride + (size_t)sg.blk * geo.upb_gu * 2 * MAT;
    return p.dn + (size_t)e * p.dn_estride + (size_t)sg.blk * geo.upb_dn * MAT;
  };

  // ================================================================ producer
  if (warp == kProdWarp) {
    uint32_t s = 0, issued = 0;
    bool ok = true;
    auto seg = [&](const Seg& sg) {
      if (lane != 0) return;
      const uint8_t* base = block_base(sg);
      const uint32_t ub = unit_bytes(sg);
      const uint32_t sc_unit = sg.list != L_DN ? 256u : 128u;   // FP8 scales of one unit
      const float* sc_base = nullptr;
      if (PER_UNIT) {
        const int e = seg_expert(p, c, sg.x);
        sc_base = sg.list != L_DN ? p.gsc + ((size_t)(e * geo.nbi + sg.blk) * geo.upb_gu) * 256
                                  : p.dsc + ((size_t)(e * geo.nbh + sg.blk) * geo.upb_dn) * 128;
      }
      const int per = stage_units(sg);
      for (int u = sg.k0; u < sg.k1; u += per) {
        const uint32_t slot = s % p.nst, q = s / p.nst;
        const uint32_t n = (uint32_t)min(per, sg.k1 - u), bytes = n * ub;
        if (ok && q > 0) ok = wait_bar(p, c, &empty[slot], (q - 1) & 1);
        if (ok) {
          mbar_arrive_expect_tx(&full[slot], bytes);
          tma_load_1d(ring + (size_t)slot * p.slot_bytes, base + (size_t)u * ub, bytes, &full[slot]);
          issued = s + 1;
          if (PER_UNIT) prefetch_l2(sc_base + (size_t)u * sc_unit, n * sc_unit * 4);   // read by the epilogue
        }
        ++s;
      }
    };
    if (lane == 0) {
      const int e0 = (int)((long long)blockIdx.x * p.E / G), e1 = (int)((long long)(blockIdx.x + 1) * p.E / G);
      prefetch_l2_span(p.router_t + (size_t)e0 * H, (size_t)(e1 - e0) * H * 4);
      prefetch_l2_span(p.norm_w, (size_t)H * (p.norm_bf16 ? 2 : 4));
      prefetch_l2_span(p.bias, (size_t)p.E * 4);
    }
    tc_segments(p, geo, L_SGU, 0, seg);
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
    uint32_t t = 0, ua = 0, ndrain = 0, nb = 0;
    int prev_x = -1;
    bool b_pending = false;
    auto warp_ok = [&](bool v) { return __shfl_sync(0xffffffffu, (int)v, 0) != 0; };
    bool ok = true;
    if (lane == 0) ok = wait_flag(p, c, &c->n_ready);
    ok = warp_ok(ok);
    const uint32_t b_addr = smem_u32(regA);
    const uint32_t idesc = umma_idesc_f16(128, 16);
    const uint32_t b_bytes = (uint32_t)I * 32u;
    const uint64_t bdesc_gu = umma_desc(b_addr, 128u, 0u), bdesc_dn = umma_desc(b_addr, 256u, 128u);
    auto acc_claim = [&]() {   // the accumulator buffer for the next tile
      const uint32_t buf = t % NACC;
      if (t >= NACC) {
        if (lane == 0 && ok) ok = wait_bar(p, c, &c->accempty[buf], ((t / NACC) - 1) & 1u);
        ok = warp_ok(ok);
      }
      tc_fence_after();
      return tmem + acc_col(buf);
    };
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
      uint32_t d0 = PER_UNIT ? 0u : acc_claim();
      for (int u = sg.k0; u < sg.k1; ++u) {
        if (PER_UNIT) d0 = acc_claim();
        const uint32_t ab = ua % kAb;
        if (lane == 0 && ok) ok = wait_bar(p, c, &c->abfull[ab], (ua / kAb) & 1u);
        ok = warp_ok(ok);
        tc_fence_after();
        if (ok) {
          // the unit's 8 K-steps (gate and up as a pair) from one elected lane
          const uint32_t a0 = tmem + kAbCol + 128u * ab;
          const int kg0 = u * kKS;   // contraction group of the B operand
          // a fresh accumulator per FP8 unit; MXFP4 adds the segment's units up
          const uint32_t acc0 = (!PER_UNIT && u > sg.k0) ? 1u : 0u;
          if (gu) umma_unit_f16(d0, a0, bdesc_gu + (uint64_t)(kg0 * 8), 16u, idesc, acc0, true);   // 2 groups of 128 B a step
          else umma_unit_f16(d0, a0, bdesc_dn + (uint64_t)(kg0 * 16), 32u, idesc, acc0, false);   // 2 groups of 256 B
        }
        umma_commit_warp(&c->abempty[ab]);
        ++ua;
        if (PER_UNIT) {
          umma_commit_warp(&c->accfull[t % NACC]);
          ++t;
        }
      }
      if (!PER_UNIT) {
        umma_commit_warp(&c->accfull[t % NACC]);
        ++t;
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
    umma_commit_warp(&c->drain);
    if (lane == 0) {
      const uint64_t t0 = globaltimer();
      while (!mbar_test(&c->drain, ndrain & 1u) && globaltimer() - t0 < p.timeout_ns) __nanosleep(64);
      while (b_pending && !mbar_test(&c->bfull, (nb - 1) & 1u) && globaltimer() - t0 < 2 * p.timeout_ns)
        __nanosleep(64);
    }
    __syncwarp();
    bar_sync(kBarEnd, 9 * 32);
    tc_fence_after();
    tmem_dealloc(tmem, kTqTmemCols);
    return;
  }

  // ================================================================ prologue
  prologue_mix(p, c, regA, ep1);
  if (warp >= kCtlWarp0) {
    control_warps(p, c, regA, ep1, false);
    return;
  }
  collapse_norm<true>(p, c, regA, ep1);
  // the router reads n as bf16 (the layer's values); the MMAs then take it
  // as fp16 (exact for normal values; below 2^-14 fp16 keeps 2^-24 steps)
  router_logits<true>(p, c, regA, false);
  {
    const int H8 = H / 8;
    for (int q = tid; q < R * H8; q += kCW * 32) {
      uint4* w = reinterpret_cast<uint4*>(regA + n_off<true>(q / H8, (q % H8) * 8, H, true));
      uint4 v = *w;
      uint32_t* u = reinterpret_cast<uint32_t*>(&v);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2 h = __floats2half2_rn(bf16lo(u[k]), bf16hi(u[k]));
        u[k] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *w = v;
    }
  }
  fence_proxy_async_smem();   // n is read by the tensor cores (async proxy)
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) *(volatile int*)&c->n_ready = 1;
  trace(p, 3, tid == 0);
  route_rows(p, c, ep1);

  // the compute warps agree on the expert list once
  if (tid == 0) {
    const bool ok = wait_flag(p, c, &c->lists_ready);
    c->nu_comp = (ok && !c->dead) ? c->nu : 0;
  }
  bar_sync(kBarCons, kCW * 32);
  const int nu = c->nu_comp;

  // ==================================================== converters, epilogue
  // Converter warp w: its lane quadrant (w & 3) of tensor memory, thread =
  // weight row.  With eight converter warps (MXFP4) warps 4-7 take the gate
  // matrix (or the first half of the chunks of a down unit) and warps 0-3
  // the up matrix (or the second half); with four (FP8), warps 4-7 take all.
  const bool converts = NCV == 8 || warp >= 4;
  const int row = (warp & 3) * 32 + lane;
  const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  uint32_t s = 0, ua = 0;
  bool cok = true;
  auto convert_units = [&](const Seg& sg) {
    const bool gu = sg.list != L_DN;
    const int per = stage_units(sg);
    for (int u0 = sg.k0; u0 < sg.k1; u0 += per) {
      const uint32_t slot = s % p.nst, q = s / p.nst;
      const int n = min(per, sg.k1 - u0);
      // lane 0 waits; the warp follows its answer (tcgen05.st is warp-wide)
      if (lane == 0 && cok) cok = wait_bar(p, c, &full[slot], q & 1);
      cok = __shfl_sync(0xffffffffu, (int)cok, 0) != 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t ab = ua % kAb;
        if (lane == 0 && ua >= kAb && cok) cok = wait_bar(p, c, &c->abempty[ab], ((ua / kAb) - 1) & 1u);
        cok = __shfl_sync(0xffffffffu, (int)(cok && !c->dead), 0) != 0;
        tc_fence_after();
        const uint8_t* st = ring + (size_t)slot * p.slot_bytes + (size_t)j * MAT;
        const uint32_t col = lane_base + kAbCol + 128u * ab;
        if (cok) {
          if (NCV == 4) {
            tq_convert<WT>(st, row, col, 0, F::CHUNKS);
            if (gu) tq_convert<WT>(st + MAT, row, col + 64u, 0, F::CHUNKS);
          } else if (gu) {
            if (warp >= 4) tq_convert<WT>(st, row, col, 0, F::CHUNKS);
            else tq_convert<WT>(st + MAT, row, col + 64u, 0, F::CHUNKS);
          } else {
            if (warp >= 4) tq_convert<WT>(st, row, col, 0, F::CHUNKS / 2);
            else tq_convert<WT>(st, row, col, F::CHUNKS / 2, F::CHUNKS);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c->abfull[ab]);
        ++ua;
      }
      if (lane == 0) mbar_arrive(&empty[slot]);   // every unit of the stage is read
      ++s;
    }
  };

  if (warp < 4) {
    // ============================================================ epilogue
    // thread <-> row i = 32 w + l of the 128-row tile (its TMEM lane)
    const int i = tid;
    uint32_t t = 0;
    bool ok = true;
    auto take = [&](uint32_t* v, uint32_t* w2) {   // the next accumulator tile
      const uint32_t buf = t % NACC;
      if (ok) ok = wait_bar(p, c, &c->accfull[buf], (t / NACC) & 1u);
      tc_fence_after();
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + acc_col(buf), v);
      tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + acc_col(buf) + 16u, w2);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c->accempty[buf]);
      ++t;
    };
    // the accumulator work of a segment (its conversion is done)
    auto finish = [&](const Seg& sg) {
      const bool gu = sg.list != L_DN;
      const int upb = gu ? geo.upb_gu : geo.upb_dn;
      float a[8], b[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) a[r] = b[r] = 0.f;
      uint32_t v[16], w2[16];
      if (PER_UNIT) {
        // FP8: scale each unit's fp32 tile by its row's block scale (the
        // producer brought the scales to L2); two units' scales in flight
        const int e = seg_expert(p, c, sg.x);
        const float* sc = gu ? p.gsc + ((size_t)(e * geo.nbi + sg.blk) * upb) * 256
                             : p.dsc + ((size_t)(e * geo.nbh + sg.blk) * upb) * 128;
        const int us = gu ? 256 : 128;
        auto ld_g = [&](int u) { return u < sg.k1 ? __ldg(sc + (size_t)u * us + i) : 0.f; };
        auto ld_u = [&](int u) { return gu && u < sg.k1 ? __ldg(sc + (size_t)u * us + 128 + i) : 0.f; };
        float sg0 = ld_g(sg.k0), su0 = ld_u(sg.k0), sg1 = ld_g(sg.k0 + 1), su1 = ld_u(sg.k0 + 1);
        for (int u = sg.k0; u < sg.k1; ++u) {
          const float sg2 = ld_g(u + 2), su2 = ld_u(u + 2);
          take(v, w2);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            if (gu) {
              a[r] = fmaf(sg0, __uint_as_float(v[r]), a[r]);
              b[r] = fmaf(su0, __uint_as_float(w2[r]), b[r]);
            } else {
              a[r] = fmaf(sg0, __uint_as_float(v[2 * r]) + __uint_as_float(v[2 * r + 1]), a[r]);
            }
          }
          sg0 = sg1;
          su0 = su1;
          sg1 = sg2;
          su1 = su2;
        }
      } else {
        take(v, w2);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          if (gu) {
            a[r] = __uint_as_float(v[r]);
            b[r] = __uint_as_float(w2[r]);
          } else {
            a[r] = __uint_as_float(v[2 * r]) + __uint_as_float(v[2 * r + 1]);
          }
        }
      }
      trace(p, 20, t == 1 && tid == 0);
      const bool live = ok && cok && !c->dead;
      if (!epi_combine(p, c, geo, sg, upb, gu, live, i, a, b)) return;
      epi_store(p, c, geo, sg, gu, live, i, a, b);
    };
    // When these warps also convert (MXFP4), a segment's accumulator work
    // waits until the next segment of the list is converted: the MMAs of
    // that segment run meanwhile (the accumulators alternate).  The last
    // segment of a list is finished before the next list starts converting
    // (a down expert may wait for this CTA's own gate/up block).
    Seg pend;
    bool has_pend = false;
    auto seg = [&](const Seg& sg) {
      if (!converts) {
        finish(sg);
        return;
      }
      convert_units(sg);
      if (has_pend) finish(pend);
      pend = sg;
      has_pend = true;
    };
    auto flush = [&]() {
      if (has_pend) finish(pend);
      has_pend = false;
    };
    tc_segments(p, geo, L_SGU, 0, seg);
    flush();
    trace(p, 6, tid == 0);
    tc_segments(p, geo, L_RGU, nu, seg);
    flush();
    trace(p, 7, tid == 0);
    tc_segments(p, geo, L_DN, nu, seg);
    flush();
    trace(p, 9, tid == 0);
    bar_sync(kBarEpi, 4 * 32);
    if (tid == 0) {
      __threadfence();
      red_release_add(&p.sync->cnt_y, 1u);
    }
    tc_fence_before();
    bar_arrive(kBarEnd, 9 * 32);   // the issuer may free the tensor memory
  } else {
    // ============================================================ converters
    tc_segments(p, geo, L_SGU, 0, convert_units);
    tc_segments(p, geo, L_RGU, nu, convert_units);
    tc_segments(p, geo, L_DN, nu, convert_units);
    tc_fence_before();
    bar_arrive(kBarEnd, 9 * 32);   // the issuer may free the tensor memory
  }

  // ==================================================================== tail
  bar_sync(kBarCons, kCW * 32);
  if (tid == 0) wait_count(p, c, &p.sync->cnt_y, ep1 * (uint32_t)G, 6u);
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
