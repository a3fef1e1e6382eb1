// kind::f8f6f4 (e4m3) tcgen05 helpers shared by the e4m3 attention kernel
// and the hardware-rate diagnostics: instruction descriptor, MMA wrappers
// (shared-memory or tensor-memory A), the issuer's four-MMA groups with a
// barrier test, and the shared-memory descriptors of the e4m3 tiles.
#pragma once
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {
namespace f8 {

// kind::f8f6f4 instruction descriptor: fp32 accumulator (bit 4), A and B
// e4m3 (format 0 in bits 7-9 and 10-12), B MN-major flag (bit 16), N >> 3
// (bits 17-22), M >> 4 (bits 24-28); A K-major, dense, no negation.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N, bool b_mn_major) {
  return (1u << 4) | ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}
// D[tmem] (+)= A[smem] * B[smem]^T, both e4m3.
__device__ __forceinline__ void mma_ss_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], A (e4m3, 4 per 32-bit column) from tensor memory.
__device__ __forceinline__ void mma_ts_e4m3(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The issuer's lookahead form of the four MMAs of a group (see mma8_ss_probe):
// a non-blocking test of the next group's K / V barrier is issued before the
// MMAs and read after them.  Step k: A and B 32 bytes (2 descriptor units)
// further along the row (S), or A 8 tensor-memory columns and B 32 keys = 4 KB
// (256 descriptor units) further (P.V).
__device__ __forceinline__ uint32_t mma4_ss_e4m3_probe(uint32_t d, uint64_t a0, uint64_t b0,
                                                       uint32_t idesc, uint32_t acc_first,
                                                       uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred t, p, one;\n\t.reg .b64 a, b;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 t, [%5], %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 one, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], %2, %3, %7, p;\n\t"
      "add.s64 a, %2, 2;\n\tadd.s64 b, %3, 2;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 4;\n\tadd.s64 b, %3, 4;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], a, b, %7, one;\n\t"
      "add.s64 a, %2, 6;\n\tadd.s64 b, %3, 6;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], a, b, %7, one;\n\t"
      "selp.u32 %0, 1, 0, t;\n\t}\n"
      : "=r"(ok)
      : "r"(d), "l"(a0), "l"(b0), "r"(acc_first), "r"(smem_u32(bar)), "r"(parity), "r"(idesc)
      : "memory");
  return ok;
}
__device__ __forceinline__ uint32_t mma4_ts_e4m3_probe(uint32_t d, uint32_t a0, uint64_t b0,
                                                       uint32_t idesc, uint32_t acc_first,
                                                       uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred t, p, one;\n\t.reg .b32 a;\n\t.reg .b64 b;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 t, [%5], %6;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.eq.b32 one, 0, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], [%2], %3, %7, p;\n\t"
      "add.u32 a, %2, 8;\n\tadd.s64 b, %3, 256;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 16;\n\tadd.s64 b, %3, 512;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], [a], b, %7, one;\n\t"
      "add.u32 a, %2, 24;\n\tadd.s64 b, %3, 768;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%1], [a], b, %7, one;\n\t"
      "selp.u32 %0, 1, 0, t;\n\t}\n"
      : "=r"(ok)
      : "r"(d), "r"(a0), "l"(b0), "r"(acc_first), "r"(smem_u32(bar)), "r"(parity), "r"(idesc)
      : "memory");
  return ok;
}
// K-major e4m3 tile: rows 128 B apart, 8-row groups 1024 B apart; step k
// (32 elements) lives 32 B further along the row.
__device__ __forceinline__ uint64_t kmajor8_desc(uint32_t tile_saddr, int k) {
  return sw128_desc(tile_saddr + uint32_t(k) * 32u, 16u, 1024u);
}
// MN-major e4m3 V tile ([keys][dims], 128 dims = one swizzle atom wide): key
// rows 128 B apart, 8-row groups 1024 B apart (SBO); step k = 32 keys = 4 KB.
// With a single atom across N the leading offset has no next atom to point
// to; it is given the minimum (16 B), which keeps any address inside the tile.
__device__ __forceinline__ uint64_t mnmajor8_desc(uint32_t tile_saddr, int k) {
  return sw128_desc(tile_saddr + uint32_t(k) * 4096u, 16u, 1024u);
}
}  // namespace f8
}  // namespace sm100
}  // namespace fkv
