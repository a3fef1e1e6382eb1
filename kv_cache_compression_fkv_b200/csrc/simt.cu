// CUDA-core (SIMT) kernels: fp32 path of segment scoring and of attention,
// and the finalisation of the segment mass (both dtypes).
//
// Frame-mode segment mass (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
// "关键模块" 3), computed in one pass over the history keys:
//   a CTA owns (layer, head, frame f, 32 scoring queries) and produces, per
//   query row i, the frame-local max m_{f,i} and sum l_{f,i} = sum_{j in f}
//   2^(z_ij - m_{f,i}) of the base-2 logits z = scale*log2(e)*q.k;
//   finalisation merges the frames of a row, M_i = max_f m_{f,i},
//   L_i = sum_f l_{f,i} 2^(m_{f,i} - M_i), and sums
//   mass_f = sum_i l_{f,i} 2^(m_{f,i} - M_i) / L_i over the rows in a fixed
//   order (deterministic, no atomics).
//
// Attention (the chunk over the compressed cache followed by its own keys):
//   a CTA owns 32 query rows of one (layer, head) and streams 32-key tiles of
//   the two key ranges through shared memory with an online softmax.
#include "fkv_internal.cuh"

namespace fkv {

constexpr int kBQ = 32;        // query rows per CTA
constexpr int kBK = 32;        // keys per shared-memory tile
constexpr int kThreads = 256;  // 8 threads per query row
constexpr int kDMax = 128;
constexpr int kLd = kDMax + 1; // padded row pitch (floats)
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// Copies rows [0, n) of a [rows][D] tile (source row r at src + r*row_stride
// elements) into shared memory as float, zero-filling rows n .. nrows-1.
template <typename T>
__device__ __forceinline__ void load_tile(float* dst, int nrows, const T* src, int64_t row_stride,
                                          int n, int D) {
  const int q4 = D / 4;
  for (int idx = threadIdx.x; idx < nrows * q4; idx += kThreads) {
    const int r = idx / q4, c = (idx - r * q4) * 4;
    float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
    if (r < n) {
      const T* p = src + int64_t(r) * row_stride + c;
      if constexpr (sizeof(T) == 4) {
        const float4 v = *reinterpret_cast<const float4*>(p);
        x0 = v.x; x1 = v.y; x2 = v.z; x3 = v.w;
      } else {
        const uint2 v = *reinterpret_cast<const uint2*>(p);
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&v.x);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&v.y);
        x0 = __low2float(a); x1 = __high2float(a); x2 = __low2float(b); x3 = __high2float(b);
      }
    }
    float* q = dst + r * kLd + c;
    q[0] = x0; q[1] = x1; q[2] = x2; q[3] = x3;
  }
}

// ---------------------------------------------------------------------------
// Segment mass, partial pass.  grid = (ceil(n_s / 32), F, L*H).

template <typename T>
__global__ void __launch_bounds__(kThreads)
score_frame_partial_kernel(int D, int T_, int F, int64_t Lq, int stride, int64_t n_s, float sl2,
                           const T* __restrict__ q_cur, const T* __restrict__ k_hist,
                           const T* __restrict__ k_cur, const uint8_t* __restrict__ head_role,
                           float2* __restrict__ part_ml) {
  const int lh = blockIdx.z;
  if (!head_role[lh]) return;
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + kBQ * kLd;
  const int f = blockIdx.y;
  const int64_t row0 = int64_t(blockIdx.x) * kBQ;
  const int nq = int(min64(kBQ, n_s - row0));
  load_tile(Qs, kBQ, q_cur + (int64_t(lh) * Lq + row0 * stride) * D, int64_t(stride) * D, nq, D);
  const int r = threadIdx.x >> 3, c8 = threadIdx.x & 7;
  float m = -INFINITY, l = 0.f;
  // f < F: history frame f; f == F: the chunk's own keys (normaliser only).
  const bool chunk = f == F;
  const T* kf = chunk ? k_cur + int64_t(lh) * Lq * D : k_hist + (int64_t(lh) * F * T_ + int64_t(f) * T_) * D;
  const int nkeys = chunk ? int(Lq) : T_;
  for (int k0 = 0; k0 < nkeys; k0 += kBK) {
    const int nk = min(kBK, nkeys - k0);
    __syncthreads();
    load_tile(Ks, kBK, kf + int64_t(k0) * D, D, nk, D);
    __syncthreads();
    float s[kBK / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int v = 0; v < kBK / 8; ++v) {
      const int j = c8 + 8 * v;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = fmaf(Qs[r * kLd + d], Ks[j * kLd + d], acc);
      s[v] = j < nk ? acc * sl2 : -INFINITY;
      tmax = fmaxf(tmax, s[v]);
    }
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
    const float mn = fmaxf(m, tmax);
    float ps = 0.f;
#pragma unroll
    for (int v = 0; v < kBK / 8; ++v) ps += exp2f(s[v] - mn);
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
    l = l * exp2f(m - mn) + ps;
    m = mn;
  }
  if (c8 == 0 && r < nq) part_ml[(int64_t(lh) * n_s + row0 + r) * (F + 1) + f] = make_float2(m, l);
}

// Frame masses from the partial statistics (layout of score_layout: F*split
// frame entries per head, split consecutive pieces per frame, then `chunk`
// entries of the chunk's own keys when they join the normaliser; G = F*split +
// chunk entries in the row normaliser):
//   frame part  (m_f, l_f) = the merge of frame f's `split` entries
//               (m_f = max m, l_f = sum l 2^(m - m_f)); the chunk's entries
//               form one more part;
//   row merge   M_i = max_f m_f,  L_i = sum_f l_f 2^(m_f - M_i)
//               (stored as (M_i, 1/L_i) in row_ml),
//   frame mass  mass_f = sum_i c_{f,i},  c_{f,i} = l_f 2^(m_f - M_i) / L_i.
// Two kernels, every sum in a fixed order (deterministic, equal frames give
// bit-equal masses):
//   score_rows_kernel    one warp per (head, row): lane t merges parts t,
//                        t + 32, ... (each read once, its entries loaded
//                        together), writes (m_f, l_f) over the part's first
//                        entry, the lanes' merges combine in a fixed shuffle
//                        tree, then each lane turns its parts into c_{f,i},
//                        written over the m of the frame's first entry (each
//                        warp touches only its own row);
//   score_frames_kernel  one CTA per (head, frame): threads stride the rows,
//                        a fixed shuffle tree and a fixed warp order.
constexpr int kRowWarps = 8;

// (m, l) of the union of two partial softmax sums; empty parts are (-inf, 0).
__device__ __forceinline__ float2 merge_part(float2 a, float2 b) {
  const float M = fmaxf(a.x, b.x);
  if (M == -INFINITY) return make_float2(-INFINITY, 0.f);
  return make_float2(M, (a.y != 0.f ? a.y * exp2f(a.x - M) : 0.f) +
                            (b.y != 0.f ? b.y * exp2f(b.x - M) : 0.f));
}

__global__ void __launch_bounds__(kRowWarps * 32)
score_rows_kernel(int F, int split, int chunk, int E, int64_t n_s,
                  const uint8_t* __restrict__ head_role, float2* __restrict__ part_ml,
                  float2* __restrict__ row_ml) {
  pdl_wait();
  const int lh = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t i = int64_t(blockIdx.x) * kRowWarps + warp;
  if (!head_role[lh] || i >= n_s) return;  // warp-uniform
  float2* p = part_ml + (int64_t(lh) * n_s + i) * E;  // the row's E entries, contiguous
  const int nparts = F + (chunk > 0 ? 1 : 0);
  // 1. each lane's parts, merged in part order
  float2 mine = make_float2(-INFINITY, 0.f);
  for (int f = lane; f < nparts; f += 32) {
    const int n = f < F ? split : chunk;
    const float2* e = p + f * split;  // the chunk part starts at F * split
    float2 part = make_float2(-INFINITY, 0.f);
    int g = 0;
    for (; g + 4 <= n; g += 4) {  // four loads in flight
      const float2 e0 = e[g], e1 = e[g + 1], e2 = e[g + 2], e3 = e[g + 3];
      part = merge_part(part, e0);
      part = merge_part(part, e1);
      part = merge_part(part, e2);
      part = merge_part(part, e3);
    }
    for (; g < n; ++g) part = merge_part(part, e[g]);
    if (f < F) p[f * split] = part;  // only this lane reads it back
    mine = merge_part(mine, part);
  }
  // 2. the row's (M, L): a fixed shuffle tree over the lanes
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float2 other = make_float2(__shfl_xor_sync(0xffffffffu, mine.x, o),
                                     __shfl_xor_sync(0xffffffffu, mine.y, o));
    mine = (lane & o) ? merge_part(other, mine) : merge_part(mine, other);
  }
  const float M = mine.x, inv = 1.f / mine.y;
  if (lane == 0) row_ml[int64_t(lh) * n_s + i] = make_float2(M, inv);
  // 3. c_{f,i} over the m of each frame's first entry
  for (int f = lane; f < F; f += 32) {
    const float2 part = p[f * split];
    p[f * split].x = part.y != 0.f ? part.y * exp2f(part.x - M) * inv : 0.f;
  }
}

// One CTA per (head, frame): thread t sums rows t, t + 256, ... in order, then
// a fixed shuffle tree per warp and the warp sums in warp order.
constexpr int kFrameThreads = 256;

__global__ void __launch_bounds__(kFrameThreads)
score_frames_kernel(int F, int split, int E, int64_t n_s, const uint8_t* __restrict__ head_role,
                    const float2* __restrict__ part_ml, float* __restrict__ seg_score,
                    const int32_t* __restrict__ poison) {
  __shared__ float wsum[kFrameThreads / 32];
  pdl_wait();
  const int f = blockIdx.x, lh = blockIdx.y;
  float* out = seg_score + int64_t(lh) * F + f;
  if (!head_role[lh]) {
    if (threadIdx.x == 0) *out = 0.f;
    return;
  }
  if (poison && *poison != 0) {  // the statistics kernel gave up: no score to give
    if (threadIdx.x == 0) *out = __int_as_float(0x7fc00000);  // NaN
    return;
  }
  const float2* cf = part_ml + int64_t(lh) * n_s * E + f * split;
  float acc = 0.f;
#pragma unroll 4
  for (int64_t i = threadIdx.x; i < n_s; i += kFrameThreads) acc += cf[i * E].x;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) wsum[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kFrameThreads / 32; ++w) t += wsum[w];
    *out = t;
  }
}

cudaError_t launch_score_frame_simt(const Dims& d, const void* q_cur, const void* k_hist,
                                    const void* k_cur, const uint8_t* head_role, float2* part_ml,
                                    cudaStream_t s) {
  const size_t smem = sizeof(float) * 2 * kBQ * kLd;
  dim3 grid(unsigned((d.n_s + kBQ - 1) / kBQ), unsigned(d.F + (d.score_with_chunk ? 1 : 0)),
            unsigned(d.LH));
  const float sl2 = d.scale * kLog2e;
  if (d.bf16)
    score_frame_partial_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
        d.D, d.T, d.F, d.Lq, d.stride, d.n_s, sl2, static_cast<const __nv_bfloat16*>(q_cur),
        static_cast<const __nv_bfloat16*>(k_hist), static_cast<const __nv_bfloat16*>(k_cur),
        head_role, part_ml);
  else
    score_frame_partial_kernel<float><<<grid, kThreads, smem, s>>>(
        d.D, d.T, d.F, d.Lq, d.stride, d.n_s, sl2, static_cast<const float*>(q_cur),
        static_cast<const float*>(k_hist), static_cast<const float*>(k_cur), head_role, part_ml);
  return cudaGetLastError();
}

cudaError_t launch_score_frame_finalize(const Dims& d, const ScoreLayout& sl,
                                        const uint8_t* head_role, float2* part_ml,
                                        float2* row_ml, float* seg_score, cudaStream_t s,
                                        const int32_t* poison) {
  if (d.n_s > 0) {
    dim3 grid(unsigned((d.n_s + kRowWarps - 1) / kRowWarps), unsigned(d.LH));
    // both finalize kernels follow this call's statistics kernel on the stream
    cudaError_t e = launch_kernel(score_rows_kernel, grid, dim3(kRowWarps * 32), 0, s, true, d.F,
                                  sl.split, sl.chunk, sl.E, d.n_s, head_role, part_ml, row_ml);
    if (e != cudaSuccess) return e;
  }
  if (d.F < 1) return cudaSuccess;
  return launch_kernel(score_frames_kernel, dim3(unsigned(d.F), unsigned(d.LH)),
                       dim3(kFrameThreads), 0, s, true, d.F, sl.split, sl.E, d.n_s, head_role,
                       static_cast<const float2*>(part_ml), seg_score, poison);
}

// ---------------------------------------------------------------------------
// Attention.  grid = (ceil(Lq / 32), L*H).

template <typename T>
__global__ void __launch_bounds__(kThreads)
attend_simt_kernel(int D, int64_t Lq, int64_t comp_rows, int64_t seg_len, int64_t max_kept,
                   float sl2, const T* __restrict__ q_cur, const T* __restrict__ k_cur,
                   const T* __restrict__ v_cur, const T* __restrict__ k_comp,
                   const T* __restrict__ v_comp, const int32_t* __restrict__ kept_cnt,
                   T* __restrict__ out) {
  extern __shared__ float smem[];
  float* Qs = smem;
  float* Ks = Qs + kBQ * kLd;
  float* Vs = Ks + kBK * kLd;
  float* Ps = Vs + kBK * kLd;  // [kBQ][kBK + 1]
  const int lh = blockIdx.y;
  const int64_t row0 = int64_t(blockIdx.x) * kBQ;
  const int nq = int(min64(kBQ, Lq - row0));
  int64_t cnt = kept_cnt[lh];
  cnt = cnt < 0 ? 0 : (cnt > max_kept ? max_kept : cnt);
  int64_t nA = cnt * seg_len;
  if (nA > comp_rows) nA = comp_rows;
  load_tile(Qs, kBQ, q_cur + (int64_t(lh) * Lq + row0) * D, D, nq, D);
  const int r = threadIdx.x >> 3, c8 = threadIdx.x & 7;
  const int nd = (D + 7) / 8;  // dims per thread: c8 + 8u < D
  float o[kDMax / 8];
#pragma unroll
  for (int u = 0; u < kDMax / 8; ++u) o[u] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int64_t tilesA = (nA + kBK - 1) / kBK;
  const int64_t tiles = tilesA + (Lq + kBK - 1) / kBK;
  for (int64_t t = 0; t < tiles; ++t) {
    const T *kp, *vp;
    int nk;
    if (t < tilesA) {
      const int64_t k0 = t * kBK;
      nk = int(min64(kBK, nA - k0));
      kp = k_comp + (int64_t(lh) * comp_rows + k0) * D;
      vp = v_comp + (int64_t(lh) * comp_rows + k0) * D;
    } else {
      const int64_t k0 = (t - tilesA) * kBK;
      nk = int(min64(kBK, Lq - k0));
      kp = k_cur + (int64_t(lh) * Lq + k0) * D;
      vp = v_cur + (int64_t(lh) * Lq + k0) * D;
    }
    __syncthreads();
    load_tile(Ks, kBK, kp, D, nk, D);
    load_tile(Vs, kBK, vp, D, nk, D);
    __syncthreads();
    float s[kBK / 8];
    float tmax = -INFINITY;
#pragma unroll
    for (int v = 0; v < kBK / 8; ++v) {
      const int j = c8 + 8 * v;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = fmaf(Qs[r * kLd + d], Ks[j * kLd + d], acc);
      s[v] = j < nk ? acc * sl2 : -INFINITY;
      tmax = fmaxf(tmax, s[v]);
    }
#pragma unroll
    for (int w = 1; w < 8; w <<= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, w));
    const float mn = fmaxf(m, tmax);
    const float corr = exp2f(m - mn);
    float ps = 0.f;
#pragma unroll
    for (int v = 0; v < kBK / 8; ++v) {
      const float p = exp2f(s[v] - mn);
      Ps[r * (kBK + 1) + c8 + 8 * v] = p;
      ps += p;
    }
#pragma unroll
    for (int w = 1; w < 8; w <<= 1) ps += __shfl_xor_sync(0xffffffffu, ps, w);
    l = l * corr + ps;
    m = mn;
    __syncwarp();
#pragma unroll
    for (int u = 0; u < kDMax / 8; ++u) {
      if (u < nd && c8 + 8 * u < D) {
        float acc = o[u] * corr;
        for (int j = 0; j < kBK; ++j) acc = fmaf(Ps[r * (kBK + 1) + j], Vs[j * kLd + c8 + 8 * u], acc);
        o[u] = acc;
      }
    }
  }
  if (r < nq) {
    T* op = out + (int64_t(lh) * Lq + row0 + r) * D;
    const float inv = 1.f / l;
#pragma unroll
    for (int u = 0; u < kDMax / 8; ++u)
      if (u < nd && c8 + 8 * u < D) op[c8 + 8 * u] = from_f32<T>(o[u] * inv);
  }
}

cudaError_t launch_attend_simt(const Dims& d, const void* q_cur, const void* k_cur,
                               const void* v_cur, const void* k_comp, const void* v_comp,
                               const int32_t* kept_cnt, void* out, cudaStream_t s) {
  const size_t smem = sizeof(float) * (kBQ * kLd + 2 * kBK * kLd + kBQ * (kBK + 1));
  dim3 grid(unsigned((d.Lq + kBQ - 1) / kBQ), unsigned(d.LH));
  const float sl2 = d.scale * kLog2e;
  cudaError_t e;
  if (d.bf16) {
    e = cudaFuncSetAttribute(attend_simt_kernel<__nv_bfloat16>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attend_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
        d.D, d.Lq, d.comp_rows, d.seg_len, d.max_kept, sl2,
        static_cast<const __nv_bfloat16*>(q_cur), static_cast<const __nv_bfloat16*>(k_cur),
        static_cast<const __nv_bfloat16*>(v_cur), static_cast<const __nv_bfloat16*>(k_comp),
        static_cast<const __nv_bfloat16*>(v_comp), kept_cnt, static_cast<__nv_bfloat16*>(out));
  } else {
    e = cudaFuncSetAttribute(attend_simt_kernel<float>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attend_simt_kernel<float><<<grid, kThreads, smem, s>>>(
        d.D, d.Lq, d.comp_rows, d.seg_len, d.max_kept, sl2, static_cast<const float*>(q_cur),
        static_cast<const float*>(k_cur), static_cast<const float*>(v_cur),
        static_cast<const float*>(k_comp), static_cast<const float*>(v_comp), kept_cnt,
        static_cast<float*>(out));
  }
  return cudaGetLastError();
}

}  // namespace fkv
