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
// Query rows: a half-warp per row, amax by shuffles, one pass.  fkv_step_fp8
// quantises the kept segments, the chunk's segments and its query rows in
// one launch.
#include <cooperative_groups.h>
#include <cuda_fp8.h>

#include "fkv_internal.cuh"

namespace cg = cooperative_groups;

namespace fkv {

constexpr int kSegCta = 8;         // CTAs per segment (one cluster)
constexpr int kSegThreads = 256;
constexpr int kSegBatch = 8;       // loads in flight per thread (4: 6% slower kept-segment gather, 13: slower)

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

// One launch quantises up to two groups of segments and, optionally, the
// query rows.  Group 0 then group 1 take the slots [0, n0) and [n0, n0 + n1);
// blockIdx.z = 0 / 1: K / V of slot blockIdx.x / kSegCta, a cluster of
// kSegCta CTAs per (slot, head, K or V); blockIdx.z = 2: query rows, CTA x of
// head lh taking rows [x q / gx, (x + 1) q / gx) of that head.  z_base = 2
// launches the query rows alone (grid.z = 1).
struct SegGroup {
  int32_t n_slots;
  int64_t src_rows, dst_rows;   // rows per head of the source and the destination
  const int32_t* kept_idx;      // gather: slot p < kept_cnt[lh] takes frame kept_idx[lh][p];
  const int32_t* kept_cnt;      // null: slot g takes frame g
  const uint4 *src_k, *src_v;
  uint2 *dst_k, *dst_v;
  float *scale_k, *scale_v;     // [LH][n_slots]
};
struct QuantPlan {
  int32_t T, vpr, F, z_base;
  SegGroup g[2];
  int64_t q_rows;               // query rows per head (plane 2)
  const uint4* q_src;
  uint2* q_dst;
  float* q_scale;               // [LH][q_rows]
  int32_t* status;
};

__global__ void __cluster_dims__(kSegCta, 1, 1) __launch_bounds__(kSegThreads)
quant_kernel(const QuantPlan p) {
  cg::cluster_group cluster = cg::this_cluster();
  __shared__ float s_part[kSegThreads / 32];
  __shared__ float s_amax;
  pdl_wait();
  const int lh = blockIdx.y;
  const int plane = int(blockIdx.z) + p.z_base;
  if (plane == 2) {
    // Query rows: a half-warp per row, lane g of it holding elements [8g, 8g+8).
    const int64_t gx = gridDim.x;
    const int64_t r_lo = p.q_rows * blockIdx.x / gx, r_hi = p.q_rows * (blockIdx.x + 1) / gx;
    const int g = threadIdx.x & 15;
    const uint4* src = p.q_src + int64_t(lh) * p.q_rows * 16;
    uint2* dst = p.q_dst + int64_t(lh) * p.q_rows * 16;
    float* scales = p.q_scale + int64_t(lh) * p.q_rows;
    for (int64_t r0 = r_lo; r0 < r_hi; r0 += kSegThreads / 16) {
      const int64_t r = r0 + (threadIdx.x >> 4);
      const bool ok = r < r_hi;
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
    return;
  }
  // Segments.  Every decision to skip depends on (lh, slot) only, so a
  // cluster skips as a whole.
  int slot = int(blockIdx.x) / kSegCta;
  const int gi = slot < p.g[0].n_slots ? 0 : 1;
  if (gi == 1) slot -= p.g[0].n_slots;
  const SegGroup& G = p.g[gi];
  if (slot >= G.n_slots) return;
  const int T_ = p.T, vpr = p.vpr;
  const int rank = int(cluster.block_rank());
  const bool is_v = plane != 0;
  int32_t f = slot;
  if (G.kept_cnt) {
    int32_t cnt = G.kept_cnt[lh];
    if (cnt < 0 || cnt > G.n_slots) {
      if (slot == 0 && rank == 0 && !is_v && threadIdx.x == 0)
        report(p.status, FKV_ERR_DEVICE_ARG, lh);
      cnt = cnt < 0 ? 0 : G.n_slots;
    }
    if (slot >= cnt) return;
    f = G.kept_idx[int64_t(lh) * G.n_slots + slot];
    if (f < 0 || f >= p.F) {
      if (rank == 0 && !is_v && threadIdx.x == 0) report(p.status, FKV_ERR_DEVICE_ARG, lh);
      return;
    }
  }
  if (int64_t(slot + 1) * T_ > G.dst_rows) {  // the destination has no room for it
    if (rank == 0 && !is_v && threadIdx.x == 0) report(p.status, FKV_ERR_DEVICE_ARG, lh);
    return;
  }
  const int64_t nvec = int64_t(T_) * vpr;
  const uint4* src = (is_v ? G.src_v : G.src_k) + (int64_t(lh) * G.src_rows + int64_t(f) * T_) * vpr;
  uint2* dst = (is_v ? G.dst_v : G.dst_k) + (int64_t(lh) * G.dst_rows + int64_t(slot) * T_) * vpr;
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
    (is_v ? G.scale_v : G.scale_k)[int64_t(lh) * G.n_slots + slot] = scale;
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

namespace {
SegGroup kept_group(const Dims& d, const int32_t* kept_idx, const int32_t* kept_cnt,
                    const void* k_hist, const void* v_hist, void* k_comp, void* v_comp,
                    float* sk, float* sv) {
  SegGroup g{};
  g.n_slots = d.F > 0 ? int32_t(d.max_kept) : 0;
  g.src_rows = d.N;
  g.dst_rows = d.comp_rows;
  g.kept_idx = kept_idx;
  g.kept_cnt = kept_cnt;
  g.src_k = static_cast<const uint4*>(k_hist);
  g.src_v = static_cast<const uint4*>(v_hist);
  g.dst_k = static_cast<uint2*>(k_comp);
  g.dst_v = static_cast<uint2*>(v_comp);
  g.scale_k = sk;
  g.scale_v = sv;
  return g;
}
SegGroup chunk_group(const Dims& d, const void* k_cur, const void* v_cur, void* k8, void* v8,
                     float* sk, float* sv) {
  SegGroup g{};
  g.n_slots = d.Fc;
  g.src_rows = g.dst_rows = d.Lq;
  g.src_k = static_cast<const uint4*>(k_cur);
  g.src_v = static_cast<const uint4*>(v_cur);
  g.dst_k = static_cast<uint2*>(k8);
  g.dst_v = static_cast<uint2*>(v8);
  g.scale_k = sk;
  g.scale_v = sv;
  return g;
}

cudaError_t launch_plan(const Dims& d, QuantPlan p, cudaStream_t s) {
  if (d.LH < 1) return cudaSuccess;
  p.T = d.T;
  p.vpr = d.D / 8;
  p.F = d.F;
  const int64_t slots = int64_t(p.g[0].n_slots) + p.g[1].n_slots;
  const bool rows = p.q_rows > 0;
  if (slots == 0 && !rows) return cudaSuccess;
  if (slots * kSegCta > 0x7fffffff) return cudaErrorInvalidConfiguration;
  // the query rows share the segments' x extent, or take about 16 rows per
  // thread pass (x a multiple of the cluster size) when launched alone
  int64_t gx = slots * kSegCta;
  if (slots == 0) {
    gx = (p.q_rows + 4 * (kSegThreads / 16) - 1) / (4 * (kSegThreads / 16));
    gx = (gx + kSegCta - 1) / kSegCta * kSegCta;
  }
  p.z_base = slots == 0 ? 2 : 0;
  const unsigned gz = slots == 0 ? 1u : (rows ? 3u : 2u);
  return launch_kernel(quant_kernel, dim3(unsigned(gx), unsigned(d.LH), gz), dim3(kSegThreads), 0,
                       s, d.pdl, p);
}
}  // namespace

cudaError_t launch_quant_kept(const Dims& d, const int32_t* kept_idx, const int32_t* kept_cnt,
                              const void* k_hist, const void* v_hist, const fkv_fp8_cache_t& c,
                              int32_t* status, cudaStream_t s) {
  QuantPlan p{};
  p.g[0] = kept_group(d, kept_idx, kept_cnt, k_hist, v_hist, c.k_comp, c.v_comp, c.k_comp_scale,
                      c.v_comp_scale);
  p.status = status;
  return launch_plan(d, p, s);
}

cudaError_t launch_quant_chunk(const Dims& d, const void* q_cur, const void* k_cur,
                               const void* v_cur, const fkv_fp8_cache_t& c, int32_t* status,
                               cudaStream_t s) {
  QuantPlan p{};
  p.g[0] = chunk_group(d, k_cur, v_cur, c.k_cur, c.v_cur, c.k_cur_scale, c.v_cur_scale);
  p.q_rows = d.Lq;
  p.q_src = static_cast<const uint4*>(q_cur);
  p.q_dst = static_cast<uint2*>(c.q_cur);
  p.q_scale = c.q_scale;
  p.status = status;
  return launch_plan(d, p, s);
}

cudaError_t launch_quant_step(const Dims& d, const int32_t* kept_idx, const int32_t* kept_cnt,
                              const void* k_hist, const void* v_hist, const void* q_cur,
                              const void* k_cur, const void* v_cur, const fkv_fp8_cache_t& c,
                              int32_t* status, cudaStream_t s) {
  QuantPlan p{};
  p.g[0] = kept_group(d, kept_idx, kept_cnt, k_hist, v_hist, c.k_comp, c.v_comp, c.k_comp_scale,
                      c.v_comp_scale);
  p.g[1] = chunk_group(d, k_cur, v_cur, c.k_cur, c.v_cur, c.k_cur_scale, c.v_cur_scale);
  p.q_rows = d.Lq;
  p.q_src = static_cast<const uint4*>(q_cur);
  p.q_dst = static_cast<uint2*>(c.q_cur);
  p.q_scale = c.q_scale;
  p.status = status;
  return launch_plan(d, p, s);
}

}  // namespace fkv
