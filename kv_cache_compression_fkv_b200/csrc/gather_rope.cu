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
// plain compaction.
#include "fkv_internal.cuh"

namespace fkv {

constexpr int kRopeThreads = 256;
constexpr int kRopeUnroll = 4;

template <typename T>
__device__ __forceinline__ uint4 rotate_vec(uint4 raw, int first_pair, int n_pairs,
                                            const float* __restrict__ omega, float delta);

// 8 bf16 = 4 pairs per 16-byte vector.
template <>
__device__ __forceinline__ uint4 rotate_vec<__nv_bfloat16>(uint4 raw, int first_pair, int n_pairs,
                                                           const float* __restrict__ omega,
                                                           float delta) {
  uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const int i = first_pair + t;
    if (i < n_pairs) {
      const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&w[t]);
      const float x0 = __low2float(b), x1 = __high2float(b);
      float s, c;
      sincosf(omega[i] * delta, &s, &c);
      const __nv_bfloat162 r = __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
      w[t] = *reinterpret_cast<const uint32_t*>(&r);
    }
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// 4 floats = 2 pairs per 16-byte vector.
template <>
__device__ __forceinline__ uint4 rotate_vec<float>(uint4 raw, int first_pair, int n_pairs,
                                                   const float* __restrict__ omega, float delta) {
  float x[4] = {__uint_as_float(raw.x), __uint_as_float(raw.y), __uint_as_float(raw.z),
                __uint_as_float(raw.w)};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int i = first_pair + t;
    if (i < n_pairs) {
      float s, c;
      sincosf(omega[i] * delta, &s, &c);
      const float x0 = x[2 * t], x1 = x[2 * t + 1];
      x[2 * t] = x0 * c - x1 * s;
      x[2 * t + 1] = x0 * s + x1 * c;
    }
  }
  return make_uint4(__float_as_uint(x[0]), __float_as_uint(x[1]), __float_as_uint(x[2]),
                    __float_as_uint(x[3]));
}

template <typename T>
__global__ void __launch_bounds__(kRopeThreads)
gather_rope_kernel(int32_t T_, int32_t F, int32_t comp_rows, int32_t vec_per_row,
                   int32_t n_pairs, const float* __restrict__ omega,
                   const uint4* __restrict__ k_hist, const uint4* __restrict__ v_hist,
                   const int32_t* __restrict__ kept_idx, const int32_t* __restrict__ kept_cnt,
                   uint4* __restrict__ k_comp, uint4* __restrict__ v_comp, int32_t* status) {
  constexpr int kPairsPerVec = 8 / int(sizeof(T));  // bf16: 4, fp32: 2
  const int lh = blockIdx.y;
  int32_t cnt = kept_cnt[lh];
  if (cnt < 0 || cnt > F) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    cnt = cnt < 0 ? 0 : F;
  }
  int64_t rows = int64_t(cnt) * T_;
  if (rows > comp_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    rows = comp_rows;
  }
  const int64_t nvec = rows * vec_per_row;
  const int32_t* kidx = kept_idx + int64_t(lh) * F;
  const int64_t hist_rows = int64_t(F) * T_;
  const uint4* ks = k_hist + int64_t(lh) * hist_rows * vec_per_row;
  const uint4* vs = v_hist + int64_t(lh) * hist_rows * vec_per_row;
  uint4* kd = k_comp + int64_t(lh) * comp_rows * vec_per_row;
  uint4* vd = v_comp + int64_t(lh) * comp_rows * vec_per_row;
  const int64_t step = int64_t(gridDim.x) * kRopeThreads * kRopeUnroll;
  for (int64_t base = int64_t(blockIdx.x) * kRopeThreads * kRopeUnroll + threadIdx.x;
       base < nvec; base += step) {
    uint4 kv[kRopeUnroll], vv[kRopeUnroll];
    int64_t dst[kRopeUnroll];
    float dlt[kRopeUnroll];
    int fp[kRopeUnroll];
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      const int64_t i = base + int64_t(u) * kRopeThreads;
      dst[u] = -1;
      if (i < nvec) {
        const int32_t r = int32_t(i / vec_per_row);
        const int32_t v = int32_t(i - int64_t(r) * vec_per_row);
        const int32_t p = r / T_;
        const int32_t f = kidx[p];
        if (f >= 0 && f < F) {
          const int64_t src = (int64_t(f) * T_ + (r - p * T_)) * vec_per_row + v;
          kv[u] = __ldcs(ks + src);
          vv[u] = __ldcs(vs + src);
          dst[u] = i;
          dlt[u] = float((F - cnt + p) - f);
          fp[u] = v * kPairsPerVec;
        } else {
          report(status, FKV_ERR_DEVICE_ARG, lh);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kRopeUnroll; ++u) {
      if (dst[u] >= 0) {
        const uint4 k = fp[u] < n_pairs ? rotate_vec<T>(kv[u], fp[u], n_pairs, omega, dlt[u]) : kv[u];
        __stcs(kd + dst[u], k);
        __stcs(vd + dst[u], vv[u]);
      }
    }
  }
}

cudaError_t launch_gather_rope(const Dims& d, const void* k_hist, const void* v_hist,
                               const int32_t* kept_idx, const int32_t* kept_cnt,
                               const float* omega, int32_t n_pairs, void* k_comp, void* v_comp,
                               int32_t* status, cudaStream_t s) {
  const int vec_per_row = d.D * d.elem / 16;
  const int64_t per_block = int64_t(kRopeThreads) * kRopeUnroll;
  const int64_t rows_max = d.comp_rows < d.N ? d.comp_rows : d.N;
  int64_t bx = (rows_max * vec_per_row + per_block - 1) / per_block;
  if (bx < 1) bx = 1;
  if (bx > 65535) bx = 65535;
  dim3 grid(unsigned(bx), unsigned(d.LH));
  if (d.bf16)
    gather_rope_kernel<__nv_bfloat16><<<grid, kRopeThreads, 0, s>>>(
        d.T, d.F, int32_t(d.comp_rows), vec_per_row, n_pairs, omega,
        static_cast<const uint4*>(k_hist), static_cast<const uint4*>(v_hist), kept_idx, kept_cnt,
        static_cast<uint4*>(k_comp), static_cast<uint4*>(v_comp), status);
  else
    gather_rope_kernel<float><<<grid, kRopeThreads, 0, s>>>(
        d.T, d.F, int32_t(d.comp_rows), vec_per_row, n_pairs, omega,
        static_cast<const uint4*>(k_hist), static_cast<const uint4*>(v_hist), kept_idx, kept_cnt,
        static_cast<uint4*>(k_comp), static_cast<uint4*>(v_comp), status);
  return cudaGetLastError();
}

}  // namespace fkv
