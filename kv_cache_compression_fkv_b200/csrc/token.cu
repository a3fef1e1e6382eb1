// Token variant, step 2: participative scores (Deep Forcing,
// bxzpzcl.cn/news/2125000, section 3.1 step 2): phi_j = sum_r q_r . k_j over
// the scoring queries r, for every candidate token j (no scale, no softmax).
//
// By linearity phi_j = qbar . k_j with qbar = sum_r q_r, so the step is a
// q-sum (fp32, in a fixed order) followed by a GEMV that reads each candidate
// key row exactly once: bound by HBM bandwidth.  The bf16 / D = 128 GEMV
// moves 16-byte vectors, 16 lanes per 256-byte row, 8 rows in flight per
// warp, with streaming (evict-first) loads.
#include "fkv_internal.cuh"

namespace fkv {

constexpr int kQsumGroups = 8;
constexpr int kQsumThreads = 128 * kQsumGroups;

// qbar[lh][d] = sum_r q_score[lh][r][d]: row groups r = g mod 8 summed in
// order, then the 8 group sums added in a fixed order (fp32 path).
template <typename T>
__global__ void __launch_bounds__(kQsumThreads)
qsum_kernel(int D, int64_t n_q, const T* __restrict__ q_score, float* __restrict__ qbar) {
  __shared__ float part[kQsumGroups][128];
  const int lh = blockIdx.x;
  const int d = threadIdx.x % 128, g = threadIdx.x / 128;
  float acc = 0.f;
  if (d < D) {
    const T* q = q_score + int64_t(lh) * n_q * D + d;
    for (int64_t r = g; r < n_q; r += kQsumGroups) acc += to_f32(q[r * D]);
  }
  part[g][d] = acc;
  __syncthreads();
  if (g == 0 && d < D) {
    float tot = 0.f;
    for (int k = 0; k < kQsumGroups; ++k) tot += part[k][d];
    qbar[int64_t(lh) * D + d] = tot;
  }
}

// bf16, D = 128: 16 threads per 256-byte row, each thread 8 dims through one
// 16-byte load per row; 64 row groups (r = g mod 64) summed in order, then
// the 64 group sums per dim added in a fixed order.
constexpr int kQsumRowGroups = 64;
#ifndef FKV_QSUM_BATCH
#define FKV_QSUM_BATCH 8
#endif
constexpr int kQsumBatch = FKV_QSUM_BATCH;
__global__ void __launch_bounds__(1024)
qsum_bf16_kernel(int64_t n_q, const uint4* __restrict__ q_score, float* __restrict__ qbar) {
  __shared__ float part[kQsumRowGroups][128];
  const int lh = blockIdx.x;
  const int sub = threadIdx.x & 15, g = threadIdx.x >> 4;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const uint4* q = q_score + int64_t(lh) * n_q * 16 + sub;
  // kQsumBatch rows of the group loaded before any is added (bytes in flight),
  // then added in row order
  for (int64_t r0 = g; r0 < n_q; r0 += int64_t(kQsumBatch) * kQsumRowGroups) {
    uint4 v[kQsumBatch];
#pragma unroll
    for (int u = 0; u < kQsumBatch; ++u) {
      const int64_t r = r0 + int64_t(u) * kQsumRowGroups;
      v[u] = r < n_q ? __ldcs(q + r * 16) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kQsumBatch; ++u) {
      if (r0 + int64_t(u) * kQsumRowGroups >= n_q) break;
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
        acc[2 * e] += __low2float(b);
        acc[2 * e + 1] += __high2float(b);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[g][sub * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < 128) {
    float tot = 0.f;
    for (int k = 0; k < kQsumRowGroups; ++k) tot += part[k][threadIdx.x];
    qbar[int64_t(lh) * 128 + threadIdx.x] = tot;
  }
}

// bf16, D = 128.  grid = (blocks per head, L*H), 256 threads.
constexpr int kPhiThreads = 256;
#ifndef FKV_PHI_CTAS_PER_SM
#define FKV_PHI_CTAS_PER_SM 8
#endif
#ifndef FKV_PHI_UNROLL
#define FKV_PHI_UNROLL 4
#endif
constexpr int kPhiUnroll = FKV_PHI_UNROLL;  // row pairs in flight per warp

__global__ void __launch_bounds__(kPhiThreads)
phi_bf16_kernel(int64_t N, int64_t S, int64_t n_c, const uint4* __restrict__ k_hist,
                const float* __restrict__ qbar, float* __restrict__ phi) {
  pdl_wait();
  const int lh = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane & 15;      // 16-byte chunk of the row: dims 8*sub .. 8*sub+7
  const int pair = lane >> 4;     // which of the warp's two rows
  float qb[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) qb[e] = qbar[int64_t(lh) * 128 + sub * 8 + e];
  const uint4* kc = k_hist + (int64_t(lh) * N + S) * 16;
  float* out = phi + int64_t(lh) * n_c;
  const int64_t warps_total = int64_t(gridDim.x) * (kPhiThreads / 32);
  const int64_t per_iter = 2 * kPhiUnroll;
  for (int64_t r0 = (int64_t(blockIdx.x) * (kPhiThreads / 32) + warp) * per_iter; r0 < n_c;
       r0 += warps_total * per_iter) {
    uint4 v[kPhiUnroll];
#pragma unroll
    for (int u = 0; u < kPhiUnroll; ++u) {
      const int64_t row = r0 + 2 * u + pair;
      v[u] = row < n_c ? __ldcs(kc + row * 16 + sub) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kPhiUnroll; ++u) {
      const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[e]);
        acc = fmaf(qb[2 * e], __low2float(b), acc);
        acc = fmaf(qb[2 * e + 1], __high2float(b), acc);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      const int64_t row = r0 + 2 * u + pair;
      if (sub == 0 && row < n_c) out[row] = acc;
    }
  }
}

// Any dtype / D (fp32 path): one warp per candidate row, lanes over D in
// 4-element groups.
template <typename T>
__global__ void phi_generic_kernel(int D, int64_t N, int64_t S, int64_t n_c,
                                   const T* __restrict__ k_hist, const float* __restrict__ qbar,
                                   float* __restrict__ phi) {
  const int lh = blockIdx.y;
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int q4 = D / 4;
  float qb[4] = {0.f, 0.f, 0.f, 0.f};
  if (lane < q4)
    for (int t = 0; t < 4; ++t) qb[t] = qbar[int64_t(lh) * D + lane * 4 + t];
  const T* kc = k_hist + (int64_t(lh) * N + S) * D;
  for (int64_t j = int64_t(blockIdx.x) * warps + (threadIdx.x >> 5); j < n_c;
       j += int64_t(gridDim.x) * warps) {
    float acc = 0.f;
    if (lane < q4) {
      const T* p = kc + j * D + lane * 4;
      for (int t = 0; t < 4; ++t) acc = fmaf(qb[t], to_f32(p[t]), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) phi[int64_t(lh) * n_c + j] = acc;
  }
}


cudaError_t launch_score_token(const Dims& d, const void* q_score, const void* k_hist,
                               float* qbar, float* seg_score, cudaStream_t s) {
  if (d.bf16)
    qsum_bf16_kernel<<<d.LH, 1024, 0, s>>>(d.n_score_q, static_cast<const uint4*>(q_score), qbar);
  else
    qsum_kernel<float><<<d.LH, kQsumThreads, 0, s>>>(d.D, d.n_score_q,
                                                     static_cast<const float*>(q_score), qbar);
  if (d.bf16) {
    // About FKV_PHI_CTAS_PER_SM CTAs of 256 threads per SM over all heads.
    int64_t per_head = (int64_t(num_sms()) * FKV_PHI_CTAS_PER_SM + d.LH - 1) / d.LH;
    const int64_t rows_per_block = (kPhiThreads / 32) * 2 * kPhiUnroll;
    const int64_t need = (d.nseg + rows_per_block - 1) / rows_per_block;
    if (per_head > need) per_head = need;
    if (per_head < 1) per_head = 1;
    dim3 grid(unsigned(per_head), unsigned(d.LH));
    // follows this call's q-sum kernel on the stream
    cudaError_t e = launch_kernel(phi_bf16_kernel, grid, dim3(kPhiThreads), 0, s, true, d.N, d.S,
                                  d.nseg, static_cast<const uint4*>(k_hist),
                                  static_cast<const float*>(qbar), seg_score);
    if (e != cudaSuccess) return e;
  } else {
    const int warps = 8;
    int64_t bx = (d.nseg + warps - 1) / warps;
    if (bx > 4096) bx = 4096;
    dim3 grid(unsigned(bx), unsigned(d.LH));
    phi_generic_kernel<float><<<grid, warps * 32, 0, s>>>(
        d.D, d.N, d.S, d.nseg, static_cast<const float*>(k_hist), qbar, seg_score);
  }
  return cudaGetLastError();
}

}  // namespace fkv
