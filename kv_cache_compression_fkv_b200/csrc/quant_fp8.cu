// e4m3 quantisation of the attention operands (the fp8 compressed cache).
//
// The Forcing-KV page says the compression composes with KV quantization
// (ai-feeds.com/i/paper/2605.09681, "与现有产品/工作流的接口" item 3) and
// fixes no format.  Here: one fp32 scale per (layer, head, segment) for K and
// for V, a segment being a kept history frame or a frame of the chunk, and one
// per query row for Q.  scale = amax / 448, code = e4m3_rn_satfinite(x *
// (448 / amax)) (scale 1 / inverse 1 for an all-zero block), every step one
// correctly rounded fp32 operation.
//
// Segments: a cluster of kSegCta CTAs per (segment, head, K or V).  Each CTA
// reduces the amax of its slice of the segment's T x D elements, the cluster
// combines the kSegCta values through distributed shared memory, then each CTA
// reads its slice again (from L2: a cluster's segment is at most a few MB and
// is read back at once) and writes the codes, 8 bf16 in -> 8 bytes out.
// Query rows: a half-warp per row, amax by shuffles, one pass.
#include <cooperative_groups.h>
#include <cuda_fp8.h>

#include "fkv_internal.cuh"

namespace cg = cooperative_groups;

namespace fkv {

constexpr int kSegCta = 8;         // CTAs per segment (one cluster)
constexpr int kSegThreads = 256;
constexpr int kSegBatch = 8;       // loads in flight per thread (4: 6% slower kept-segment gather, 13: slower)
constexpr int kRowThreads = 256;   // 16 rows of 16 lanes per CTA pass

__device__ __forceinline__ float amax8(uint4 raw) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  __nv_bfloat162 m = __habs2(h[0]);
  m = __hmax2(m, __habs2(h[1]));
  m = __hmax2(m, __habs2(h[2]));
  m = __hmax2(m, __habs2(h[3]));
  return fmaxf(__low2float(m), __high2float(m));
}

// 8 bf16 times inv, rounded once to fp32, then to e4m3 (element 0 in the low byte).
__device__ __forceinline__ uint2 quant8(uint4 raw, float inv) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 a = __bfloat1622float2(h[2 * i]);
    const float2 b = __bfloat1622float2(h[2 * i + 1]);
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(a.x, inv), __fmul_rn(a.y, inv)), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
        make_float2(__fmul_rn(b.x, inv), __fmul_rn(b.y, inv)), __NV_SATFINITE, __NV_E4M3);
    w[i] = uint32_t(lo) | (uint32_t(hi) << 16);
  }
  return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ void scale_pair(float amax, float* scale, float* inv) {
  if (amax > 0.f) {
    *scale = __fdiv_rn(amax, 448.f);
    *inv = __fdiv_rn(448.f, amax);
  } else {
    *scale = 1.f;
    *inv = 1.f;
  }
}

// grid = (kSegCta * n_slots, L*H, 2), cluster (kSegCta, 1, 1); blockIdx.z: 0 = K, 1 = V.
// Gather mode (kept_cnt != nullptr): slot p < kept_cnt[lh] takes source frame
// kept_idx[lh][p]; chunk mode: slot g takes source frame g.  The decision to
// skip a slot depends on (lh, slot) only, so a cluster skips as a whole.
__global__ void __cluster_dims__(kSegCta, 1, 1) __launch_bounds__(kSegThreads)
quant_segments_kernel(int32_t T_, int32_t vpr, int32_t n_slots, int32_t F, int64_t src_rows,
                      int64_t dst_rows, const int32_t* __restrict__ kept_idx,
                      const int32_t* __restrict__ kept_cnt, const uint4* __restrict__ src_k,
                      const uint4* __restrict__ src_v, uint2* __restrict__ dst_k,
                      uint2* __restrict__ dst_v, float* __restrict__ scale_k,
                      float* __restrict__ scale_v, int32_t* status) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float s_part[kSegThreads / 32];
  __shared__ float s_amax;
  const int lh = blockIdx.y;
  const int slot = int(blockIdx.x) / kSegCta;
  const int rank = int(cluster.block_rank());
  const bool is_v = blockIdx.z != 0;
  int32_t f = slot;
  if (kept_cnt) {
    int32_t cnt = kept_cnt[lh];
    if (cnt < 0 || cnt > n_slots) {
      if (slot == 0 && rank == 0 && !is_v && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
      cnt = cnt < 0 ? 0 : n_slots;
    }
    if (slot >= cnt) return;
    f = kept_idx[int64_t(lh) * n_slots + slot];
    if (f < 0 || f >= F) {
      if (rank == 0 && !is_v && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
      return;
    }
  }
  if (int64_t(slot + 1) * T_ > dst_rows) {  // the compressed cache has no room for it
    if (rank == 0 && !is_v && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    return;
  }
  const int64_t nvec = int64_t(T_) * vpr;
  const uint4* src = (is_v ? src_v : src_k) + (int64_t(lh) * src_rows + int64_t(f) * T_) * vpr;
  uint2* dst = (is_v ? dst_v : dst_k) + (int64_t(lh) * dst_rows + int64_t(slot) * T_) * vpr;
  const int64_t v0 = nvec * rank / kSegCta, v1 = nvec * (rank + 1) / kSegCta;

  // kSegBatch independent 16-byte loads in flight per thread in both passes
  float m = 0.f;
  for (int64_t b = v0 + threadIdx.x; b < v1; b += kSegThreads * kSegBatch) {
    uint4 r[kSegBatch];
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) {
      const int64_t i = b + int64_t(u) * kSegThreads;
      r[u] = i < v1 ? __ldg(src + i) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) m = fmaxf(m, amax8(r[u]));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = s_part[0];
    for (int w = 1; w < kSegThreads / 32; ++w) a = fmaxf(a, s_part[w]);
    s_amax = a;
  }
  cluster.sync();  // every CTA's slice amax is visible to the cluster
  float amax = 0.f;
#pragma unroll
  for (int r = 0; r < kSegCta; ++r) amax = fmaxf(amax, *cluster.map_shared_rank(&s_amax, r));
  float scale, inv;
  scale_pair(amax, &scale, &inv);
  if (rank == 0 && threadIdx.x == 0)
    (is_v ? scale_v : scale_k)[int64_t(lh) * n_slots + slot] = scale;
  for (int64_t b = v0 + threadIdx.x; b < v1; b += kSegThreads * kSegBatch) {
    uint4 r[kSegBatch];
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) {
      const int64_t i = b + int64_t(u) * kSegThreads;
      if (i < v1) r[u] = __ldcs(src + i);
    }
#pragma unroll
    for (int u = 0; u < kSegBatch; ++u) {
      const int64_t i = b + int64_t(u) * kSegThreads;
      if (i < v1) __stcs(dst + i, quant8(r[u], inv));
    }
  }
  cluster.sync();  // no CTA leaves while another may still read its s_amax
}

// Rows of D = 16 * 8 elements: lane g of a 16-lane group holds elements [8g, 8g+8).
__global__ void __launch_bounds__(kRowThreads)
quant_rows_kernel(int64_t rows, const uint4* __restrict__ src, uint2* __restrict__ dst,
                  float* __restrict__ scales) {
  const int g = threadIdx.x & 15;
  const int64_t step = int64_t(gridDim.x) * (kRowThreads / 16);
  for (int64_t r0 = int64_t(blockIdx.x) * (kRowThreads / 16); r0 < rows; r0 += step) {
    const int64_t r = r0 + (threadIdx.x >> 4);
    const bool ok = r < rows;
    const uint4 raw = ok ? __ldcs(src + r * 16 + g) : make_uint4(0, 0, 0, 0);
    float m = amax8(raw);
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o, 16));
    float scale, inv;
    scale_pair(m, &scale, &inv);
    if (ok) {
      __stcs(dst + r * 16 + g, quant8(raw, inv));
      if (g == 0) scales[r] = scale;
    }
  }
}

cudaError_t launch_quant_segments(const Dims& d, int n_slots, int64_t src_rows, int64_t dst_rows,
                                  const int32_t* kept_idx, const int32_t* kept_cnt,
                                  const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                                  float* scale_k, float* scale_v, int32_t* status,
                                  cudaStream_t s) {
  if (n_slots < 1 || d.LH < 1) return cudaSuccess;
  if (int64_t(n_slots) * kSegCta > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const int vpr = d.D / 8;
  dim3 grid(unsigned(n_slots * kSegCta), unsigned(d.LH), 2u);
  quant_segments_kernel<<<grid, kSegThreads, 0, s>>>(
      d.T, vpr, n_slots, d.F, src_rows, dst_rows, kept_idx, kept_cnt,
      static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
      static_cast<uint2*>(dst_k), static_cast<uint2*>(dst_v), scale_k, scale_v, status);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows(const Dims& d, const void* src, void* dst, float* scales,
                              cudaStream_t s) {
  const int64_t rows = int64_t(d.LH) * d.Lq;
  if (rows < 1) return cudaSuccess;
  int64_t blocks = (rows + kRowThreads / 16 - 1) / (kRowThreads / 16);
  const int64_t cap = int64_t(num_sms()) * 8;
  if (blocks > cap) blocks = cap;
  quant_rows_kernel<<<unsigned(blocks), kRowThreads, 0, s>>>(
      rows, static_cast<const uint4*>(src), static_cast<uint2*>(dst), scales);
  return cudaGetLastError();
}

}  // namespace fkv
