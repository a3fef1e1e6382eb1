// Compaction with temporal RoPE re-positioning of the kept keys (Deep
// Forcing, bxzpzcl.cn/news/2125000, section 2.2.2; section 3.2 item 3 applies
// the same adjustment to selected tokens).
//
// Frame mode: the p-th of cnt kept frames of a head moves from frame
// kept_idx[p] to frame F - cnt + p (the kept frames close up and end right
// before the chunk at frame F).  Its keys' temporal band -- the first n_pairs
// pairs of adjacent dims (k[2i], k[2i+1]) read as complex numbers -- is
// rotated by the angle omega[i] * delta, delta = (F - cnt + p) - kept_idx[p];
// the other dims and all values are copied unchanged.  Rotation in fp32,
// rounded once to the activation dtype.  Same 16-byte streaming copy as the
// plain compaction; each CTA stays inside one kept frame so the frame's
// cos/sin values are evaluated once per CTA.
#include "fkv_internal.cuh"

namespace fkv {

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;
constexpr int kRopeChunk = kRopeThreads * kRopeUnroll;  // 16-byte vectors per CTA
constexpr int kMaxRopePairs = 64;                       // head_dim <= 128

// cs[i] = (cos, sin) of pair i's angle for this CTA's frame.
template <typename T>
__device__ __forceinline__ uint4 rotate_vec(uint4 raw, int first_pair, int n_pairs,
                                            const float2* cs);

// 8 bf16 = 4 pairs per 16-byte vector.
template <>
__device__ __forceinline__ uint4 rotate_vec<__nv_bfloat16>(uint4 raw, int first_pair, int n_pairs,
                                                           const float2* cs) {
  uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int i = first_pair + t;
    if (i < n_pairs) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[t]);
      const float x0 = __low2float(b), x1 = __high2float(b);
      const float2 r = cs[i];
      const __nv_bfloat162 o = __floats2bfloat162_rn(x0 * r.x - x1 * r.y, x0 * r.y + x1 * r.x);
      w[t] = *reinterpret_cast<const uint32_t*>(&o);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 floats = 2 pairs per 16-byte vector.
template <>
__device__ __forceinline__ uint4 rotate_vec<float>(uint4 raw, int first_pair, int n_pairs,
                                                   const float2* cs) {
  float x[4] = {__uint_as_float(raw.x), __uint_as_float(raw.y), __uint_as_float(raw.z),
                __uint_as_float(raw.w)};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int i = first_pair + t;
    if (i < n_pairs) {
      const float2 r = cs[i];
      const float x0 = x[2 * t], x1 = x[2 * t + 1];
      x[2 * t] = x0 * r.x - x1 * r.y;
      x[2 * t + 1] = x0 * r.y + x1 * r.x;
    }
  }
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                    __float_as_uint(x[3]));
}

// One CTA copies a slice of kRopeChunk 16-byte vectors of ONE kept frame p:
// the frame's T rows are contiguous at both ends, and its rotation angles
// depend on (p, pair) only, so they are computed once per CTA into shared
// memory instead of once per element.  grid = (F * chunks_per_frame, L*H).
template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
gather_rope_kernel(int32_t T_, int32_t F, int32_t comp_rows, int32_t vec_per_row,
                   int32_t chunks_per_frame, int32_t n_pairs, const float* __restrict__ omega,
                   const uint4* __restrict__ k_hist, const uint4* __restrict__ v_hist,
                   const int32_t* __restrict__ kept_idx, const int32_t* __restrict__ kept_cnt,
                   uint4* __restrict__ k_comp, uint4* __restrict__ v_comp, int32_t* status) {
  constexpr int kPairsPerVec = 8 / int(sizeof(T));  // bf16: 4, fp32: 2
  __shared__ float2 cs[kMaxRopePairs];
  const int lh = blockIdx.y;
  const int32_t p = int32_t(blockIdx.x) / chunks_per_frame;
  const int32_t c = int32_t(blockIdx.x) - p * chunks_per_frame;
  int32_t cnt = kept_cnt[lh];
  if (cnt < 0 || cnt > F) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    cnt = cnt < 0 ? 0 : F;
  }
  if (int64_t(cnt) * T_ > comp_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
  }
  if (p >= cnt) return;
  const int32_t f = kept_idx[int64_t(lh) * F + p];
  if (f < 0 || f >= F) {
    if (threadIdx.x == 0 && c == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    return;
  }
  // destination rows of this frame, clipped to the compressed cache
  int64_t row_end = int64_t(p + 1) * T_;
  if (row_end > comp_rows) row_end = comp_rows;
  const int64_t frame_vec = (row_end - int64_t(p) * T_) * vec_per_row;
  const int64_t j0 = int64_t(c) * kRopeChunk;
  if (j0 >= frame_vec) return;
  const int64_t j1 = j0 + kRopeChunk < frame_vec ? j0 + kRopeChunk : frame_vec;
  const float delta = float((F - cnt + p) - f);
  for (int i = threadIdx.x; i < n_pairs; i += kRopeThreads) {
    float sn, cn;
    sincosf(omega[i] * delta, &sn, &cn);
    cs[i] = make_float2(cn, sn);
  }
  __syncthreads();
  const int64_t hist_rows = int64_t(F) * T_;
  const uint4* ks = k_hist + (int64_t(lh) * hist_rows + int64_t(f) * T_) * vec_per_row;
  const uint4* vs = v_hist + (int64_t(lh) * hist_rows + int64_t(f) * T_) * vec_per_row;
  uint4* kd = k_comp + (int64_t(lh) * comp_rows + int64_t(p) * T_) * vec_per_row;
  uint4* vd = v_comp + (int64_t(lh) * comp_rows + int64_t(p) * T_) * vec_per_row;
  uint4 kv[kRopeUnroll], vv[kRopeUnroll];
#pragma unroll
  for (int u = 0; u < kRopeUnroll; ++u) {
    const int64_t j = j0 + threadIdx.x + int64_t(u) * kRopeThreads;
    if (j < j1) {
      kv[u] = __ldcs(ks + j);
      vv[u] = __ldcs(vs + j);
    }
  }
#pragma unroll
  for (int u = 0; u < kRopeUnroll; ++u) {
    const int64_t j = j0 + threadIdx.x + int64_t(u) * kRopeThreads;
    if (j < j1) {
      const int32_t first = int32_t(j % vec_per_row) * kPairsPerVec;
      const uint4 k = first < n_pairs ? rotate_vec<T>(kv[u], first, n_pairs, cs) : kv[u];
      __stcs(kd + j, k);
      __stcs(vd + j, vv[u]);
    }
  }
}

cudaError_t launch_gather_rope(const Dims& d, const void* k_hist, const void* v_hist,
                               const int32_t* kept_idx, const int32_t* kept_cnt,
                               const float* omega, int32_t n_pairs, void* k_comp, void* v_comp,
                               int32_t* status, cudaStream_t s) {
  if (n_pairs > kMaxRopePairs) return cudaErrorInvalidValue;
  const int vec_per_row = d.D * d.elem / 16;
  const int64_t chunks = (int64_t(d.T) * vec_per_row + kRopeChunk - 1) / kRopeChunk;
  // at least one CTA, so that a bad kept_cnt is still reported when F == 0
  const int64_t bx = d.F > 0 ? int64_t(d.F) * chunks : 1;
  if (bx > int64_t(0x7fffffff)) return cudaErrorInvalidConfiguration;
  dim3 grid(unsigned(bx), unsigned(d.LH));
  if (d.bf16)
    gather_rope_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, s>>>(
        d.T, d.F, int32_t(d.comp_rows), vec_per_row, int32_t(chunks), n_pairs, omega,
        static_cast<const uint4*>(k_hist), static_cast<const uint4*>(v_hist), kept_idx, kept_cnt,
        static_cast<uint4*>(k_comp), static_cast<uint4*>(v_comp), status);
  else
    gather_rope_kernel<float><<<grid, kRopeThreads, 0, s>>>(
        d.T, d.F, int32_t(d.comp_rows), vec_per_row, int32_t(chunks), n_pairs, omega,
        static_cast<const uint4*>(k_hist), static_cast<const uint4*>(v_hist), kept_idx, kept_cnt,
        static_cast<uint4*>(k_comp), static_cast<uint4*>(v_comp), status);
  return cudaGetLastError();
}

}  // namespace fkv
