// Comparison selectors: uniform eviction and random drop at the same budget
// as the method (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
// "与基线对比及工程启示", first item, names both as the heuristics it beats).
// Every head keeps k_per_head[lh] segments whatever its role:
//   uniform: segments floor(i * n / k), i < k;
//   random:  the k segments of largest priority u(seed; lh, s), ties to the
//            lower index, where u = top 24 bits of the first word of
//            Philox4x64-10 (Salmon et al., SC 2011) at counter (s, lh, 0, 0),
//            key (seed, 0), scaled to [0, 1).  The priorities are written to
//            seg_score and ranked by the method's own top-k kernels.
// Token granularity: sink [0, S) and recent [N - R, N) are kept whole; the
// selectors act on the n = N - S - R candidates between them.
#include "fkv_internal.cuh"

namespace fkv {

// Philox4x64 multipliers and Weyl key increments (Salmon et al., 2011).
constexpr uint64_t kPhM0 = 0xD2E7470EE14C6C93ull, kPhM1 = 0xCA5A826395121157ull;
constexpr uint64_t kPhW0 = 0x9E3779B97F4A7C15ull, kPhW1 = 0xBB67AE8584CAA73Bull;

__device__ __forceinline__ uint64_t philox4x64_10_word0(uint64_t c0, uint64_t c1, uint64_t c2,
                                                        uint64_t c3, uint64_t k0, uint64_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += kPhW0;
      k1 += kPhW1;
    }
    const uint64_t hi0 = __umul64hi(kPhM0, c0), lo0 = kPhM0 * c0;
    const uint64_t hi1 = __umul64hi(kPhM1, c2), lo1 = kPhM1 * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  return c0;
}

__global__ void priority_kernel(int64_t total, int64_t nseg, uint64_t seed,
                                float* __restrict__ seg_score) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const uint64_t lh = uint64_t(i / nseg), s = uint64_t(i % nseg);
    const uint64_t w = philox4x64_10_word0(s, lh, 0, 0, seed, 0);
    seg_score[i] = float(uint32_t(w >> 40)) * 5.9604644775390625e-8f;  // * 2^-24, exact
  }
}

// Uniform eviction.  kept_idx row length max_kept; segments are frames (frame
// mode) or candidate tokens offset by S with sink and recent around them.
__global__ void uniform_kernel(int64_t n, int64_t S, int64_t R, int64_t max_kept,
                               const int32_t* __restrict__ k_per_head,
                               int32_t* __restrict__ kept_idx, int32_t* __restrict__ kept_cnt,
                               int32_t* status) {
  const int lh = blockIdx.x;
  int64_t k = k_per_head[lh];
  if (k < 0 || k > n) {
    if (threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    k = k < 0 ? 0 : n;
  }
  int32_t* out = kept_idx + int64_t(lh) * max_kept;
  const int64_t total = S + k + R;
  for (int64_t t = threadIdx.x; t < total; t += blockDim.x) {
    int64_t v;
    if (t < S)
      v = t;
    else if (t < S + k)
      v = S + ((t - S) * n) / k;
    else
      v = S + n + (t - S - k);  // recent: N - R + (t - S - k)
    out[t] = int32_t(v);
  }
  if (threadIdx.x == 0) kept_cnt[lh] = int32_t(total);
}

cudaError_t launch_heuristic(const Dims& d, int32_t policy, uint64_t seed,
                             const int32_t* k_per_head, float* seg_score, int32_t* kept_idx,
                             int32_t* kept_cnt, int32_t* status, cudaStream_t s) {
  const int64_t n = d.nseg;  // frames, or candidate tokens
  if (policy == FKV_POLICY_UNIFORM) {
    uniform_kernel<<<d.LH, 256, 0, s>>>(n, d.S, d.R, d.max_kept, k_per_head, kept_idx, kept_cnt,
                                        status);
    return cudaGetLastError();
  }
  const int64_t total = int64_t(d.LH) * n;
  if (total > 0) {
    int64_t blocks = (total + 255) / 256;
    const int64_t cap = int64_t(num_sms()) * 8;
    if (blocks > cap) blocks = cap;
    priority_kernel<<<unsigned(blocks), 256, 0, s>>>(total, n, seed, seg_score);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (d.token) return launch_select_token(d, seg_score, k_per_head, kept_idx, kept_cnt, status, s);
  // every head ranked (no head roles, no static masks)
  return launch_select_frame(d, seg_score, nullptr, nullptr, k_per_head, kept_idx, kept_cnt,
                             status, s);
}

}  // namespace fkv
