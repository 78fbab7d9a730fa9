// Thin inline-PTX wrappers for sm_100a: mbarriers, 1-D TMA bulk copies and
// L2 prefetch, acquire/release on global words, the global timer, and the
// hardware FP8 / FP4 pair converters.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace mono {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// one non-blocking probe of the phase with the given parity
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// one potentially blocking probe: the thread may wait in hardware for the
// phase (up to a system-dependent limit) instead of polling
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on bar
__device__ __forceinline__ void tma_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// one cache line to L2 through the load path
__device__ __forceinline__ void prefetch_l2_line(const void* src) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(src) : "memory");
}

// L2 prefetch of the 16-byte granules inside [src, src + bytes)
__device__ __forceinline__ void prefetch_l2_span(const void* src, size_t bytes) {
  const uintptr_t a = ((uintptr_t)src + 15) & ~(uintptr_t)15;
  const uintptr_t e = ((uintptr_t)src + bytes) & ~(uintptr_t)15;
  for (uintptr_t q = a; q < e; q += 65536) {
    const uintptr_t n = e - q < 65536 ? e - q : 65536;
    prefetch_l2(reinterpret_cast<const void*>(q), (uint32_t)n);
  }
}

// 16-byte asynchronous copy global -> shared (L2 only), grouped by commit
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ uint32_t ld_relaxed(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Programmatic dependent launch: wait until the grids this launch depends on
// have completed and their memory is visible (a no-op when launched without
// the attribute), and let the next grid in the stream begin its launch
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// two e4m3 codes (low byte first) -> two floats
__device__ __forceinline__ float2 e4m3x2_to_f2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

// two e2m1 codes (low nibble first) -> two floats
__device__ __forceinline__ float2 e2m1x2_to_f2(uint32_t byte) {
  uint32_t h;
  asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}\n" : "=r"(h) : "r"(byte));
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  return __half22float2(hh);
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float round_bf16(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

}  // namespace mono

namespace mono {

// ------------------------------------------------ 5th-gen tensor cores --
// Shared-memory matrix descriptor of a K-major operand without swizzle: core
// matrices of 8 rows x 16 bytes stored contiguously (128 bytes); lbo = byte
// distance between core matrices adjacent along K, sbo = along M/N.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version of sm_100
  return d;                 // base offset 0, layout SWIZZLE_NONE
}

// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, both
// K-major, M = m, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int m, int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// One tcgen05.mma (kind::f16) from a converged warp: one elected lane issues
// (the same lane every time, so its commits track all of its MMAs); the
// operands stay warp-uniform, which keeps the descriptor arithmetic cheap.
// acc: accumulate into D (else overwrite).
__device__ __forceinline__ void umma_bf16_warp(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p, e;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
      " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(acc)
      : "memory");
}
// Arrive once on bar when every tcgen05 operation the elected lane issued so
// far is complete (from a converged warp).
__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
      " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f8f6f4: e4m3 A and B (format code 0 in both
// fields), fp32 accumulator, both K-major, M = m, N = n.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// One 128 x 128 e4m3 unit from shared memory, issued by one elected lane of
// a converged warp: 4 K-steps of 32 (kind::f8f6f4), the first overwriting D.
// A advances 4096 bytes a K-step (256 descriptor units), B db_step units.
// pair: a second A matrix (up) 16384 bytes on, into d + 16.
__device__ __forceinline__ void umma_unit_e4m3(uint32_t d, uint64_t da, uint64_t db, uint32_t db_step, uint32_t idesc,
                                               bool pair) {
  if (pair) {
    asm volatile(
        "{\n .reg .pred e, t, f;\n .reg .b32 rx, d1;\n .reg .b64 a0, a1, b;\n"
        " elect.sync rx|e, 0xffffffff;\n setp.eq.b32 t, 0, 0;\n setp.ne.b32 f, 0, 0;\n"
        " mov.b64 a0, %1;\n add.u64 a1, %1, 1024;\n add.u32 d1, %0, 16;\n mov.b64 b, %2;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, f;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [d1], a1, b, %4, f;\n"
        " add.u64 a0, a0, 256;\n add.u64 a1, a1, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [d1], a1, b, %4, t;\n"
        " add.u64 a0, a0, 256;\n add.u64 a1, a1, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [d1], a1, b, %4, t;\n"
        " add.u64 a0, a0, 256;\n add.u64 a1, a1, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [d1], a1, b, %4, t;\n"
        "}\n" ::"r"(d), "l"(da), "l"(db), "l"((uint64_t)db_step), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred e, t, f;\n .reg .b32 rx;\n .reg .b64 a0, b;\n"
        " elect.sync rx|e, 0xffffffff;\n setp.eq.b32 t, 0, 0;\n setp.ne.b32 f, 0, 0;\n"
        " mov.b64 a0, %1;\n mov.b64 b, %2;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, f;\n"
        " add.u64 a0, a0, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        " add.u64 a0, a0, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        " add.u64 a0, a0, 256;\n add.u64 b, b, %3;\n"
        " @e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], a0, b, %4, t;\n"
        "}\n" ::"r"(d), "l"(da), "l"(db), "l"((uint64_t)db_step), "r"(idesc)
        : "memory");
  }
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns: thread l of the warp reads its
// quadrant's lane l
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored with the
// 128-byte swizzle (rows of 128 bytes, the 16-byte chunks of row r at chunk
// index c ^ (r % 8), 8-row atoms of 1024 bytes): sbo = byte distance between
// 8-row groups; the leading offset is unused for this layout (encoded 1).
// The atom must sit on a 1024-byte boundary; moving along K inside it adds
// the byte offset to the start address.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t sbo) {
  uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;   // descriptor version of sm_100
  d |= (uint64_t)2 << 61;   // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::mxf8f6f4 with block scales: e2m1 A, e4m3 B,
// e8m0 scale factors, fp32 accumulator, both K-major, M = m, N = n; the
// scale-factor byte selectors (bits 4-5 for B, 29-30 for A) are added per
// K-step.
__host__ __device__ constexpr uint32_t umma_idesc_mx_e2m1_e4m3(int m, int n) {
  return (5u << 7) | (0u << 10) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((uint32_t)(m >> 4) << 24);
}

// One 128 x 128 unit of e2m1 weights (A, 128-byte-swizzled K-major, in
// shared memory) against e4m3 B, block-scaled: 4 MMAs of K = 32.  The unit's
// 4 x 128 e8m0 A scales are first copied from shared memory (sfd, a chunk of
// 512 bytes) to tensor memory at sfa by tcgen05.cp (32x128b, all four lane
// quarters); K-step j then reads byte j there.  B's scales are at sfb: with
// bstep set, K-step j reads byte j (a scale per K-block), else every K-step
// reads byte bsel (one scale for the unit).  acc: the first K-step adds to D
// (else it overwrites D).  pair: a second A (up) 16384 bytes on, its scales
// from sfd2 to sfa2, into d + 16.  One elected lane of a converged warp issues
// all of it, in order.
__device__ __forceinline__ void umma_unit_mx(uint32_t d, uint64_t da, uint64_t db, uint32_t db_step, uint32_t idesc,
                                             uint32_t sfa, uint64_t sfd, uint32_t sfa2, uint64_t sfd2, uint32_t sfb,
                                             bool bstep, uint32_t bsel, bool acc, bool pair) {
  // per K-step: A scale byte +1 (idesc bits 29-30, address bits 30-31); B
  // scale byte +1 when bstep (idesc bits 4-5, address bits 30-31)
  const uint32_t istep = 0x20000000u | (bstep ? 0x10u : 0u);
  const uint32_t bastep = bstep ? 0x40000000u : 0u;
  const uint32_t i0 = idesc | ((bstep ? 0u : bsel) << 4);
  const uint32_t b0 = sfb | ((bstep ? 0u : bsel) << 30);
  if (pair) {
    asm volatile(
        "{\n .reg .pred e, t, f;\n .reg .b32 rx, d1, i, s0, s1, sb;\n .reg .b64 a0, a1, b;\n"
        " elect.sync rx|e, 0xffffffff;\n setp.eq.b32 t, 0, 0;\n setp.ne.b32 f, %11, 0;\n"
        " @e tcgen05.cp.cta_group::1.32x128b.warpx4 [%5], %6;\n"
        " @e tcgen05.cp.cta_group::1.32x128b.warpx4 [%7], %8;\n"
        " mov.b64 a0, %1;\n add.u64 a1, %1, 1024;\n add.u32 d1, %0, 16;\n mov.b64 b, %2;\n"
        " mov.b32 i, %4;\n mov.b32 s0, %5;\n mov.b32 s1, %7;\n mov.b32 sb, %9;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], f;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [d1], a1, b, i, [s1], [sb], f;\n"
        " add.u64 a0, a0, 2;\n add.u64 a1, a1, 2;\n add.u64 b, b, %3;\n"
        " add.u32 i, i, %10;\n add.u32 s0, s0, 0x40000000;\n add.u32 s1, s1, 0x40000000;\n add.u32 sb, sb, %12;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [d1], a1, b, i, [s1], [sb], t;\n"
        " add.u64 a0, a0, 2;\n add.u64 a1, a1, 2;\n add.u64 b, b, %3;\n"
        " add.u32 i, i, %10;\n add.u32 s0, s0, 0x40000000;\n add.u32 s1, s1, 0x40000000;\n add.u32 sb, sb, %12;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [d1], a1, b, i, [s1], [sb], t;\n"
        " add.u64 a0, a0, 2;\n add.u64 a1, a1, 2;\n add.u64 b, b, %3;\n"
        " add.u32 i, i, %10;\n add.u32 s0, s0, 0x40000000;\n add.u32 s1, s1, 0x40000000;\n add.u32 sb, sb, %12;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [d1], a1, b, i, [s1], [sb], t;\n"
        "}\n" ::"r"(d), "l"(da), "l"(db), "l"((uint64_t)db_step), "r"(i0), "r"(sfa), "l"(sfd), "r"(sfa2), "l"(sfd2),
        "r"(b0), "r"(istep), "r"((uint32_t)acc), "r"(bastep)
        : "memory");
  } else {
    asm volatile(
        "{\n .reg .pred e, t, f;\n .reg .b32 rx, i, s0, sb;\n .reg .b64 a0, b;\n"
        " elect.sync rx|e, 0xffffffff;\n setp.eq.b32 t, 0, 0;\n setp.ne.b32 f, %9, 0;\n"
        " @e tcgen05.cp.cta_group::1.32x128b.warpx4 [%5], %6;\n"
        " mov.b64 a0, %1;\n mov.b64 b, %2;\n mov.b32 i, %4;\n mov.b32 s0, %5;\n mov.b32 sb, %7;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], f;\n"
        " add.u64 a0, a0, 2;\n add.u64 b, b, %3;\n add.u32 i, i, %8;\n add.u32 s0, s0, 0x40000000;\n"
        " add.u32 sb, sb, %10;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        " add.u64 a0, a0, 2;\n add.u64 b, b, %3;\n add.u32 i, i, %8;\n add.u32 s0, s0, 0x40000000;\n"
        " add.u32 sb, sb, %10;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        " add.u64 a0, a0, 2;\n add.u64 b, b, %3;\n add.u32 i, i, %8;\n add.u32 s0, s0, 0x40000000;\n"
        " add.u32 sb, sb, %10;\n"
        " @e tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], a0, b, i, [s0], [sb], t;\n"
        "}\n" ::"r"(d), "l"(da), "l"(db), "l"((uint64_t)db_step), "r"(i0), "r"(sfa), "l"(sfd), "r"(b0),
        "r"(istep), "r"((uint32_t)acc), "r"(bastep)
        : "memory");
  }
}

// tcgen05.cp of one 512-byte scale chunk (32 rows x 16 bytes in shared memory)
// to 4 tensor-memory columns at taddr in every lane quarter, by one elected
// lane of a converged warp
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sfd) {
  asm volatile(
      "{\n .reg .pred e;\n .reg .b32 rx;\n elect.sync rx|e, 0xffffffff;\n"
      " @e tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n}\n" ::"r"(taddr),
      "l"(sfd)
      : "memory");
}

// 32 lanes x 4 consecutive 32-bit columns from registers (thread l of the
// warp writes its quadrant's lane l)
__device__ __forceinline__ void tmem_st4(uint32_t taddr, uint32_t v0, uint32_t v1, uint32_t v2, uint32_t v3) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(v0), "r"(v1), "r"(v2),
               "r"(v3)
               : "memory");
}

// 2-D tiled TMA load of the box at coordinates (c0, c1) of the tensor map
// into this CTA's shared memory, completion counted on bar
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// tcgen05.ld of 32 lanes x 16 columns without the wait (pair it with
// tmem_ld_wait before the registers are used)
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void bar_arrive(int id, int threads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace mono
