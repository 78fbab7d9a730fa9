// CUDA-core variant of the persistent kernel: each compute warp owns one
// weight row (or gate/up row pair) of a ring stage, lanes split the
// contraction, products in fp32 pairs (FFMA2), dequantisation in registers.
// It serves every expert format and is the only path for fp32 experts.
#pragma once
#include "common.cuh"

namespace mono {

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

// --------------------------------------------------------------- the kernel --

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) mono_ffn_cc_kernel(const __grid_constant__ Params p) {
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

  // launched behind another grid of the stream (programmatic dependent
  // launch), this grid may be resident before that one has finished: nothing
  // it wrote is read before this point
  grid_dep_wait();
  if (tid == 0) {
    // both grid words in flight at once, used after the barrier set-up
    const uint32_t ep0 = ld_relaxed(&p.sync->cnt_done);
    const uint32_t abort0 = ld_relaxed(&p.err->abort);
    c->dead = 0;
    c->lists_ready = 0;
    c->nu = 0;
    for (int s = 0; s < p.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    c->epoch = ep0;
    c->live = live_rows(p);
    if (abort0) c->dead = 1;   // fail-stop after an unreported error
    fence_barrier_init();
  }
  __syncthreads();
  grid_dep_launch();   // the next layer's grid may take each SM as this grid leaves it
  if (c->dead) return;
  const uint32_t ep1 = c->epoch + (uint32_t)G;   // every grid counter's target in this launch
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

  if (warp == kMmaWarp) return;

  prologue_mix(p, c, regA, ep1);
  if (warp >= kCtlWarp0) {
    control_warps(p, c, regA, ep1, true);
    return;
  }

  // ================================================ compute warps from here
  const int ctid = tid;   // 0..255
  collapse_norm<false>(p, c, regA, ep1);
  const void* n_s = regA;
  trace(p, 3, ctid == 0);
  router_logits<false>(p, c, regA, false);

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
    if (may_publish(p, c->epoch, 4, 4)) {
      red_release_add(&p.sync->cnt_act, 1u);
    }
    wait_count(p, c, &p.sync->cnt_act, ep1, 4u);
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

  tail(p, c, [&](int r, int h) { return ys[r * p.ymax + (h - h0)]; });
  bar_sync(kBarCons, kCW * 32);
  trace(p, 10, ctid == 0);
  finish_step(p, c, ep1);
}

}  // namespace mono
