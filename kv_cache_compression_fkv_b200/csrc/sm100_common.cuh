// Blackwell (sm_100a) building blocks written as inline PTX: mbarriers with
// bounded waits, TMA tile loads, tcgen05 MMA / commit / TMEM load-store, and
// the shared-memory and instruction descriptors of kind::f16 MMAs.
//
// Operand layout used everywhere: a [128 rows][128 bf16] tile lives in shared
// memory as two 16 KB regions (elements 0-63 and 64-127 of each row), each
// region 128 rows x 128 bytes in the 128-byte-swizzle pattern that TMA writes
// (16-byte chunk c of row r stored at chunk c ^ (r & 7)), regions aligned to
// 1024 bytes.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace fkv {
namespace sm100 {

constexpr uint32_t kTileBytes = 128 * 128 * 2;    // one [128][128] bf16 tile
constexpr uint32_t kRegionBytes = 128 * 128;      // [128 rows][64 bf16]
// Bounded waits: about one second at the B200's clocks, then the kernel gives up.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
#ifndef FKV_WAIT_HINT_NS
#define FKV_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
#if FKV_WAIT_HINT_NS > 0
  // Suspend (up to the hint) until the phase completes instead of spinning,
  // leaving issue slots to the other warps of the sub-partition.
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "n"(FKV_WAIT_HINT_NS)
      : "memory");
#else
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
#endif
  return ok != 0;
}
// Non-blocking test of the phase of the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase of the given parity to complete.  Gives up (returns
// false) when *abort is set by another thread or after `limit` cycles (by
// default kWaitCycles), in which case it sets *abort itself so that every
// role of the CTA winds down.  A phase that has already completed is seen by
// a non-blocking test.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          long long limit = kWaitCycles) {
  if (mbar_test_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      *abort = 1;
      return false;
    }
  }
}

// ---- TMA ----------------------------------------------------------------------
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}
// 3-D tiled load into shared memory, completion counted in bytes on `bar`.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* m, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}
// Both 64-column halves of a [128][128] tile starting at row `row` of slab `slab`.
__device__ __forceinline__ void tma_load_tile(uint8_t* dst, const CUtensorMap* m, uint64_t* bar,
                                              int row, int slab) {
  tma_load_3d(dst, m, bar, 0, row, slab);
  tma_load_3d(dst + kRegionBytes, m, bar, 64, row, slab);
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05 ------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, M=128, kind::f16 (bf16 in, fp32 accumulate).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], A read from tensor memory (M rows = lanes).
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Eight kind::f16 MMAs into D (K = 8 x 16; the first accumulates only when
// acc_first != 0) with a non-blocking test of an mbarrier phase placed before
// them in the same instruction stream and read only after the eighth, so the
// test's shared-memory round trip overlaps the MMA issue.  Returns 1 when the
// phase of the given parity had completed at the time of the test.  The
// operand addresses of step k are formed inside from the step-0 ones, so the
// issuing thread keeps few registers live.
//   mma8_ss_probe: A and B K-major in shared memory, both advancing as
//                  kmajor_desc does (32 B per step, the next 64-element
//                  region after step 3);
//   mma8_ts_probe: A from tensor memory (8 columns per step), B MN-major in
//                  shared memory (2048 B per step).
__device__ __forceinline__ uint32_t mma8_ss_probe(uint32_t d, uint64_t a0, uint64_t b0,
                                                  uint32_t idesc, uint32_t acc_first,
                                                  uint64_t* bar, uint32_t parity) {
  static_assert(kRegionBytes >> 4 == 1024, "descriptor step of the second region");
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred t, p, one;\n\t.reg .b64 a, b;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 t, [%5], %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 one, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], %2, %3, %7, p;\n\t"
      "add.s64 a, %2, 2;\n\tadd.s64 b, %3, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 4;\n\tadd.s64 b, %3, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 6;\n\tadd.s64 b, %3, 6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 1024;\n\tadd.s64 b, %3, 1024;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 1026;\n\tadd.s64 b, %3, 1026;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 1028;\n\tadd.s64 b, %3, 1028;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 1030;\n\tadd.s64 b, %3, 1030;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], a, b, %7, one;\n\t"
      "selp.u32 %0, 1, 0, t;\n\t}\n"
      : "=r"(ok)
      : "r"(d), "l"(a0), "l"(b0), "r"(acc_first), "r"(smem_u32(bar)), "r"(parity), "r"(idesc)
      : "memory");
  return ok;
}
__device__ __forceinline__ uint32_t mma8_ts_probe(uint32_t d, uint32_t a0, uint64_t b0,
                                                  uint32_t idesc, uint32_t acc_first,
                                                  uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred t, p, one;\n\t.reg .b32 a;\n\t.reg .b64 b;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 t, [%5], %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 one, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [%2], %3, %7, p;\n\t"
      "add.u32 a, %2, 8;\n\tadd.s64 b, %3, 128;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 16;\n\tadd.s64 b, %3, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 24;\n\tadd.s64 b, %3, 384;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 32;\n\tadd.s64 b, %3, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 40;\n\tadd.s64 b, %3, 640;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 48;\n\tadd.s64 b, %3, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 56;\n\tadd.s64 b, %3, 896;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%1], [a], b, %7, one;\n\t"
      "selp.u32 %0, 1, 0, t;\n\t}\n"
      : "=r"(ok)
      : "r"(d), "r"(a0), "l"(b0), "r"(acc_first), "r"(smem_u32(bar)), "r"(parity), "r"(idesc)
      : "memory");
  return ok;
}

// Arrives once on `bar` when every MMA issued so far by this thread is done.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 consecutive 32-bit columns of this thread's TMEM lane (warp-collective).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---- descriptors ----------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle: start address, leading
// and stride byte offsets (all >> 4), version 1 (bit 46), layout 2 (bits 61-63).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}
// K-major operand: rows 128 B apart, 8-row groups 1024 B apart; step k (16
// elements) lives 32 B further along the row, the second 64-element half in
// the next region.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int k) {
  return sw128_desc(tile_saddr + uint32_t(k >> 2) * kRegionBytes + uint32_t(k & 3) * 32u, 16u,
                    1024u);
}
// MN-major B operand (V as [keys][dims]): N (dims) contiguous within a
// 64-element region, the next 64 dims one region (LBO) further; K (keys) 128 B
// per row, 8-row groups 1024 B apart (SBO); step k = 16 keys = 2048 B.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile_saddr, int k) {
  return sw128_desc(tile_saddr + uint32_t(k) * 2048u, kRegionBytes, 1024u);
}
// Instruction descriptor of kind::f16: fp32 accumulator (bit 4), A and B bf16
// (bits 7 and 10), B MN-major flag (bit 16), N >> 3 (bits 17-22), M >> 4
// (bits 24-28); A K-major, no negation, dense.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 lanes per instruction (Blackwell packed fp32 FMA / add).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fadd2_rm(float2 a, float2 b) {  // rounded toward -inf
  uint64_t r;
  asm("add.rm.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t r;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(r)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&r);
}

// 2^x on the FMA pipe (no MUFU): Cody-Waite split x = n + f with n = floor(x)
// and f in [0, 1); 2^f from a degree-3 minimax polynomial (max relative error
// 8.6e-5 on [0, 1]; coefficients fitted by fit_exp2_poly.py beside this file,
// p(0) = 1 exactly); 2^n added to the exponent field.  floor(x) comes from
// adding 1.5*2^23 rounded toward -inf, which leaves it in the low mantissa
// bits; shifting those bits by 23 yields n << 23 modulo 2^32.  x is clamped
// to >= -127 so that -inf gives exactly +0.  Valid for x <= 127.
#ifndef FKV_POLY_DEG
#define FKV_POLY_DEG 3
#endif
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  const float kMagic = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 mg = make_float2(kMagic, kMagic);
  const float2 y = fadd2_rm(x, mg);
  const float2 f = fsub2(x, fsub2(y, mg));
#if FKV_POLY_DEG == 2
  // degree-2 fit: max relative error 2.05e-3 on [0, 1]
  const float c1 = __uint_as_float(0x3f2a7c6au);  // 6.659609079e-01
  const float c2 = __uint_as_float(0x3ea8ece9u);  // 3.299324811e-01
  float2 p = ffma2(make_float2(c2, c2), f, make_float2(c1, c1));
#else
  const float c1 = __uint_as_float(0x3f31f335u);  // 6.951172948e-01
  const float c2 = __uint_as_float(0x3e691b63u);  // 2.276435345e-01
  const float c3 = __uint_as_float(0x3d9dd5d8u);  // 7.706803083e-02
  float2 p = ffma2(make_float2(c3, c3), f, make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
#endif
  p = ffma2(p, f, make_float2(1.f, 1.f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(y.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(y.y) << 23)));
}

// Three-input maximum.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

}  // namespace sm100

// Host: 3-D bf16 tensor map of a [slabs][rows][128] array, box [1][128][64],
// 128-byte swizzle, out-of-range rows read as zero.  Returns false on error.
bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t slabs,
                    uint64_t row_stride_bytes, uint64_t slab_stride_bytes);
// Host: the same for 1-byte elements (e4m3 codes): [slabs][rows][128] bytes,
// box [1][128][128], one 128-byte swizzle atom per row.
bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t slabs,
                  uint64_t row_stride_bytes, uint64_t slab_stride_bytes);

}  // namespace fkv
