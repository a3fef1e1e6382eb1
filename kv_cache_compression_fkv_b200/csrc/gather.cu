// Step 4: compaction of the kept segments into the dense compressed cache
// (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "输出与工程收益": the pruned
// KV replaces the original cache inside attention).
//
// A pure copy, bound by HBM bandwidth.  Destination row r of head (l, h)
// belongs to kept segment r / seg_len and comes from history row
// kept_idx[r / seg_len] * seg_len + r % seg_len.  Rows are moved as 16-byte
// vectors: every thread issues all of its loads (K and V, several vectors)
// before its stores so that enough bytes are in flight per SM, loads and
// stores bypass L1 and are marked streaming (evict-first) since each byte is
// touched exactly once.
#include "fkv_internal.cuh"

namespace fkv {

constexpr int kGatherThreads = 256;
constexpr int kGatherUnroll = 4;

__global__ void __launch_bounds__(kGatherThreads)
gather_kernel(int32_t seg_len, int32_t nseg_total, int32_t max_kept, int32_t comp_rows,
              int32_t vec_per_row, int64_t hist_rows, const uint4* __restrict__ k_hist,
              const uint4* __restrict__ v_hist, const int32_t* __restrict__ kept_idx,
              const int32_t* __restrict__ kept_cnt, uint4* __restrict__ k_comp,
              uint4* __restrict__ v_comp, int32_t* status) {
  pdl_wait();
  const int lh = blockIdx.y;
  int32_t cnt = kept_cnt[lh];
  if (cnt < 0 || cnt > max_kept) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    cnt = cnt < 0 ? 0 : max_kept;
  }
  int64_t rows = int64_t(cnt) * seg_len;
  if (rows > comp_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    rows = comp_rows;
  }
  const int64_t nvec = rows * vec_per_row;
  const int32_t* kidx = kept_idx + int64_t(lh) * max_kept;
  const uint4* ks = k_hist + int64_t(lh) * hist_rows * vec_per_row;
  const uint4* vs = v_hist + int64_t(lh) * hist_rows * vec_per_row;
  uint4* kd = k_comp + int64_t(lh) * comp_rows * vec_per_row;
  uint4* vd = v_comp + int64_t(lh) * comp_rows * vec_per_row;
  const int64_t step = int64_t(gridDim.x) * kGatherThreads * kGatherUnroll;
  for (int64_t base = int64_t(blockIdx.x) * kGatherThreads * kGatherUnroll + threadIdx.x;
       base < nvec; base += step) {
    uint4 kv[kGatherUnroll], vv[kGatherUnroll];
    int64_t dst[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int64_t i = base + int64_t(u) * kGatherThreads;
      dst[u] = -1;
      if (i < nvec) {
        const int32_t r = int32_t(i / vec_per_row);
        const int32_t v = int32_t(i - int64_t(r) * vec_per_row);
        const int32_t seg = r / seg_len;
        const int32_t src_seg = kidx[seg];
        if (src_seg >= 0 && src_seg < nseg_total) {
          const int64_t src = (int64_t(src_seg) * seg_len + (r - seg * seg_len)) * vec_per_row + v;
          kv[u] = __ldcs(ks + src);
          vv[u] = __ldcs(vs + src);
          dst[u] = i;
        } else {
          report(status, FKV_ERR_DEVICE_ARG, lh);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      if (dst[u] >= 0) {
        __stcs(kd + dst[u], kv[u]);
        __stcs(vd + dst[u], vv[u]);
      }
    }
  }
}

cudaError_t launch_gather(const Dims& d, const void* k_hist, const void* v_hist,
                          const int32_t* kept_idx, const int32_t* kept_cnt, void* k_comp,
                          void* v_comp, int32_t* status, cudaStream_t s) {
  const int vec_per_row = d.D * d.elem / 16;
  const int64_t per_block = int64_t(kGatherThreads) * kGatherUnroll;
  int64_t rows_max = d.comp_rows < d.max_kept * d.seg_len ? d.comp_rows : d.max_kept * d.seg_len;
  int64_t bx = (rows_max * vec_per_row + per_block - 1) / per_block;
  if (bx < 1) bx = 1;
  if (bx > 65535) bx = 65535;
  dim3 grid(unsigned(bx), unsigned(d.LH));
  return launch_kernel(gather_kernel, grid, dim3(kGatherThreads), 0, s, d.pdl,
                       int32_t(d.seg_len), int32_t(d.seg_len == 1 ? d.N : d.F),
                       int32_t(d.max_kept), int32_t(d.comp_rows), vec_per_row, d.N,
                       static_cast<const uint4*>(k_hist), static_cast<const uint4*>(v_hist),
                       kept_idx, kept_cnt, static_cast<uint4*>(k_comp),
                       static_cast<uint4*>(v_comp), status);
}

// Next history cache: rows [0, keep*seg_len) of the output are the last
// `keep` kept segments of the compressed cache, rows after them the chunk's
// own rows.  grid = (blocks, L*H); same 16-byte streaming copy as above.
__global__ void __launch_bounds__(kGatherThreads)
advance_kernel(int32_t seg_len, int32_t max_kept, int32_t comp_rows, int32_t keep,
               int32_t chunk_rows, int32_t vec_per_row, const uint4* __restrict__ k_comp,
               const uint4* __restrict__ v_comp, const int32_t* __restrict__ kept_cnt,
               const uint4* __restrict__ k_cur, const uint4* __restrict__ v_cur,
               uint4* __restrict__ k_next, uint4* __restrict__ v_next, int32_t* status) {
  const int lh = blockIdx.y;
  int32_t cnt = kept_cnt[lh];
  bool bad = cnt < keep || cnt > max_kept || int64_t(cnt) * seg_len > comp_rows;
  if (bad && blockIdx.x == 0 && threadIdx.x == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
  const int64_t old_rows = int64_t(keep) * seg_len;
  const int64_t out_rows = old_rows + chunk_rows;
  const int64_t nvec = out_rows * vec_per_row;
  const int64_t src0 = bad ? 0 : (int64_t(cnt) - keep) * seg_len;  // first kept row copied
  const uint4* kc = k_comp + int64_t(lh) * comp_rows * vec_per_row;
  const uint4* vc = v_comp + int64_t(lh) * comp_rows * vec_per_row;
  const uint4* kn = k_cur + int64_t(lh) * chunk_rows * vec_per_row;
  const uint4* vn = v_cur + int64_t(lh) * chunk_rows * vec_per_row;
  uint4* kd = k_next + int64_t(lh) * out_rows * vec_per_row;
  uint4* vd = v_next + int64_t(lh) * out_rows * vec_per_row;
  const int64_t step = int64_t(gridDim.x) * kGatherThreads * kGatherUnroll;
  for (int64_t base = int64_t(blockIdx.x) * kGatherThreads * kGatherUnroll + threadIdx.x;
       base < nvec; base += step) {
    uint4 kv[kGatherUnroll], vv[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int64_t i = base + int64_t(u) * kGatherThreads;
      if (i < nvec) {
        const int64_t r = i / vec_per_row, v = i - r * vec_per_row;
        if (r < old_rows) {
          if (bad) {  // not enough kept segments: leave zeros, error recorded
            kv[u] = vv[u] = make_uint4(0, 0, 0, 0);
          } else {
            kv[u] = __ldcs(kc + (src0 + r) * vec_per_row + v);
            vv[u] = __ldcs(vc + (src0 + r) * vec_per_row + v);
          }
        } else {
          kv[u] = __ldcs(kn + (r - old_rows) * vec_per_row + v);
          vv[u] = __ldcs(vn + (r - old_rows) * vec_per_row + v);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const int64_t i = base + int64_t(u) * kGatherThreads;
      if (i < nvec) {
        __stcs(kd + i, kv[u]);
        __stcs(vd + i, vv[u]);
      }
    }
  }
}

cudaError_t launch_advance(const Dims& d, int64_t out_segments, const void* k_comp,
                           const void* v_comp, const int32_t* kept_cnt, const void* k_cur,
                           const void* v_cur, void* k_next, void* v_next, int32_t* status,
                           cudaStream_t s) {
  const int vec_per_row = d.D * d.elem / 16;
  const int64_t chunk_segs = d.Lq / d.seg_len;
  const int64_t keep = out_segments - chunk_segs;
  const int64_t out_rows = out_segments * d.seg_len;
  const int64_t per_block = int64_t(kGatherThreads) * kGatherUnroll;
  int64_t bx = (out_rows * vec_per_row + per_block - 1) / per_block;
  if (bx < 1) bx = 1;
  if (bx > 65535) bx = 65535;
  dim3 grid(unsigned(bx), unsigned(d.LH));
  advance_kernel<<<grid, kGatherThreads, 0, s>>>(
      int32_t(d.seg_len), int32_t(d.max_kept), int32_t(d.comp_rows), int32_t(keep),
      int32_t(d.Lq), vec_per_row, static_cast<const uint4*>(k_comp),
      static_cast<const uint4*>(v_comp), kept_cnt, static_cast<const uint4*>(k_cur),
      static_cast<const uint4*>(v_cur), static_cast<uint4*>(k_next), static_cast<uint4*>(v_next),
      status);
  return cudaGetLastError();
}

}  // namespace fkv
