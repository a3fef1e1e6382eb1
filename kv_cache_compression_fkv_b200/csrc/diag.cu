// Hardware-rate diagnostics behind the attention kernel's design: how fast
// one thread can issue tcgen05.mma of the attention's shapes, and how fast
// one or more warps of a sub-partition can run ex2 on MUFU.  Both run one CTA
// per SM and report cycles measured with clock64 by CTA 0; they touch no
// caller data.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"
#include "f8_common.cuh"

namespace fkv {
namespace sm100 {

constexpr int kDiagThreads = 384;
constexpr uint32_t kDiagSmem = 3 * 32768 + 1024;  // A 32 KB + B 64 KB, 1 KB alignment slack

// Shapes (bf16, M = 128, K = 16 per MMA, fp32 accumulator in tensor memory):
//   0  A, B K-major in shared memory, N = 128 (the Q.K^T step)
//   1  A from tensor memory, B MN-major in shared memory, N = 128 (the P.V
//      step: V stored [keys][dims])
//   2  as 0 with N = 256        3  as 0 with N = 64
//   4  as 0 with an MN-major B  5  as 1 with a K-major B
//   6  as 0, 7  as 1, issued in groups of eight through the attention
//      kernel's own issue helpers (mma8_ss_probe, mma8_ts_probe)
//   8  kind::f8f6f4 (e4m3) M128 N128 K32, A and B K-major in shared memory
//      (the e4m3 attention's Q.K^T), 9  e4m3 with A from tensor memory and
//      an MN-major B (its P.V); both in groups of four through the e4m3
//      kernel's issue helpers.  An e4m3 K32 MMA is as many FLOPs as two bf16
//      K16 ones, at twice the nominal rate: 64 cycles.
//   10 as 0 with M = 64 (a 64-row query tile: half the rows of shape 0)
// Shapes 0-5 issue straight-line code with compile-time operand offsets, so
// the issue loop holds nothing but the MMAs and their address arithmetic.
template <int kShape>
__device__ __forceinline__ void issue8(uint32_t tm, uint64_t da, uint64_t db, uint64_t dv,
                                       uint64_t* probe_bar, uint32_t da_base, uint32_t db_base) {
  // operands stay inside A [0, 32 KB) and B [32 KB, 96 KB) of the shared
  // buffer; accumulators and the tensor-memory A inside the 512 columns
  constexpr uint32_t kKOff[8] = {0, 2, 4, 6, 1024, 1026, 1028, 1030};  // K-major steps
  if constexpr (kShape == 8) {
    // e4m3 tiles: A [0, 16 KB), B [32 KB, 48 KB); step k = 32 B (K-major) or
    // 4 KB (MN-major), four steps per group
    const uint64_t a8 = f8::kmajor8_desc(uint32_t(da_base), 0), b8 = f8::kmajor8_desc(uint32_t(db_base), 0);
    for (int g = 0; g < 2; ++g)
      (void)f8::mma4_ss_e4m3_probe(tm, a8, b8, f8::idesc_e4m3(128, 128, false), 1u, probe_bar, 0u);
  } else if constexpr (kShape == 9) {
    const uint64_t v8 = f8::mnmajor8_desc(uint32_t(db_base), 0);
    for (int g = 0; g < 2; ++g)
      (void)f8::mma4_ts_e4m3_probe(tm + 384, tm + 256, v8, f8::idesc_e4m3(128, 128, true), 1u,
                                   probe_bar, 0u);
  } else if constexpr (kShape == 6) {
    (void)mma8_ss_probe(tm, da, db, idesc_bf16(128, 128, false), 1u, probe_bar, 0u);
  } else if constexpr (kShape == 7) {
    (void)mma8_ts_probe(tm + 384, tm + 256, dv, idesc_bf16(128, 128, true), 1u, probe_bar, 0u);
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      if constexpr (kShape == 0 || kShape == 2 || kShape == 3)
        mma_ss(tm, da + kKOff[k], db + kKOff[k],
               idesc_bf16(128, kShape == 2 ? 256 : kShape == 3 ? 64 : 128, false), 1u);
      else if constexpr (kShape == 10)
        mma_ss(tm, da + kKOff[k], db + kKOff[k], idesc_bf16(64, 128, false), 1u);
      else if constexpr (kShape == 1)
        mma_ts(tm + 384, tm + 256 + 8 * k, dv + 128u * k, idesc_bf16(128, 128, true), 1u);
      else if constexpr (kShape == 4)
        mma_ss(tm, da + kKOff[k], dv + 128u * k, idesc_bf16(128, 128, true), 1u);
      else
        mma_ts(tm + 384, tm + 256 + 8 * k, db + kKOff[k], idesc_bf16(128, 128, false), 1u);
    }
  }
}

// Warp 0's lane 0 issues n MMAs (n / 8 groups) back to back into one
// accumulator, then commits; with busy != 0 two other warps of its
// sub-partition run an FMA + MUFU loop meanwhile.  cycles[0] = issue time of
// the n MMAs, cycles[1] = until their completion.
template <int kShape>
__global__ void __launch_bounds__(kDiagThreads, 1)
mma_rate_kernel(int n, int busy, long long* cycles, int32_t* status) {
  extern __shared__ __align__(1024) uint8_t smraw[];
  uint8_t* sm = align1024(smraw);
  __shared__ uint64_t bar, probe_bar;
  __shared__ uint32_t tbase;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 3 * 32768 / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);  // finite operands
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init(&probe_bar, 1);  // never arrived on: the probes see it pending
    abort_flag = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(&tbase, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = tbase;
  if (warp == 0) {
    if (lane == 0) {
      const uint64_t da = kmajor_desc(smem_u32(sm), 0), db = kmajor_desc(smem_u32(sm + 32768), 0);
      const uint64_t dv = mnmajor_desc(smem_u32(sm + 32768), 0);
      const long long t0 = clock64();
      for (int i = 0; i < n; i += 8)
        issue8<kShape>(tm, da, db, dv, &probe_bar, smem_u32(sm), smem_u32(sm + 32768));
      const long long t1 = clock64();
      mma_commit(&bar);
      const bool ok = mbar_wait(&bar, 0, &abort_flag);
      const long long t2 = clock64();
      if (blockIdx.x == 0) {
        cycles[0] = t1 - t0;
        cycles[1] = t2 - t0;
      }
      if (!ok) report(status, FKV_ERR_TIMEOUT, blockIdx.x);
    }
  } else if (busy && (warp == 4 || warp == 8)) {  // the issuer's sub-partition
    float x = threadIdx.x * 1e-3f, acc = 0.f;
    for (int i = 0; i < 4096; ++i) {
      x = fmaf(x, 0.999f, 1e-4f);
      acc += ex2(x);
    }
    if (acc == 1234.5f) cycles[2] = 1;  // keeps the loop
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
}

// `warps` warps per sub-partition (warps w < 4 * warps) each run n ex2 in 8
// independent chains; cycles[0] = CTA 0, warp 0's time.
__global__ void __launch_bounds__(512, 1) ex2_rate_kernel(int n, int warps, long long* cycles) {
  const int warp = threadIdx.x >> 5;
  float x[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) x[k] = -1e-3f * float(threadIdx.x + k);
  __syncthreads();
  const long long t0 = clock64();
  if (warp < 4 * warps) {
    for (int i = 0; i < n; i += 8) {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = ex2(x[k]) - 1.0f;
    }
  }
  const long long t1 = clock64();
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) s += x[k];
  if (s == 1234.5f) cycles[1] = 1;  // keeps the chains
  if (threadIdx.x == 0 && blockIdx.x == 0) cycles[0] = t1 - t0;
}

}  // namespace sm100

cudaError_t launch_diag_mma_rate(int shape, int n, int busy, long long* cycles, int32_t* status,
                                 cudaStream_t s) {
  using namespace sm100;
  void (*const kernels[11])(int, int, long long*, int32_t*) = {
      mma_rate_kernel<0>, mma_rate_kernel<1>, mma_rate_kernel<2>, mma_rate_kernel<3>,
      mma_rate_kernel<4>, mma_rate_kernel<5>, mma_rate_kernel<6>, mma_rate_kernel<7>,
      mma_rate_kernel<8>, mma_rate_kernel<9>, mma_rate_kernel<10>};
  if (shape < 0 || shape > 10) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(kernels[shape], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(kDiagSmem));
  if (e != cudaSuccess) return e;
  kernels[shape]<<<num_sms(), kDiagThreads, kDiagSmem, s>>>(n, busy, cycles, status);
  return cudaGetLastError();
}

cudaError_t launch_diag_ex2_rate(int n, int warps, long long* cycles, cudaStream_t s) {
  sm100::ex2_rate_kernel<<<num_sms(), 512, 0, s>>>(n, warps, cycles);
  return cudaGetLastError();
}

}  // namespace fkv
