// Steps 1 and 3: kept segment lists.
//
// Frame mode (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "关键模块" 2 and 3):
//   static heads keep the frames of their fixed mask; dynamic heads keep the k
//   frames of largest score.  One CTA per (layer, head), one thread per frame:
//   each thread ranks its frame against all others under the total order
//   (score desc, index asc) and keeps it when rank < k; kept frames are then
//   written in ascending order through a ballot/popcount prefix sum.
//
// Token mode (Deep Forcing, bxzpzcl.cn/news/2125000, section 3.1 steps 1-3):
//   sink [0, S) and recent [N-R, N) are kept whole; the candidates keep their
//   C best tokens.  One CTA per (layer, head): a most-significant-digit radix
//   select over order-preserving 32-bit keys (4 passes of 8 bits) finds the
//   C-th largest key t and how many keys equal to t are taken; a stable
//   block-wide compaction then emits the chosen ids in ascending order.
#include "fkv_internal.cuh"

namespace fkv {

__global__ void select_frame_kernel(int F, const float* __restrict__ seg_score,
                                    const uint8_t* __restrict__ head_role,
                                    const uint8_t* __restrict__ static_mask,
                                    const int32_t* __restrict__ k_per_head,
                                    int32_t* __restrict__ kept_idx,
                                    int32_t* __restrict__ kept_cnt, int32_t* status) {
  extern __shared__ uint32_t keys[];
  __shared__ int warp_counts[32];
  pdl_wait();
  const int lh = blockIdx.x;
  const int f = threadIdx.x;
  const bool dyn = head_role ? head_role[lh] != 0 : true;  // no roles: every head ranked
  int k = 0;
  if (dyn) {
    k = k_per_head[lh];
    if (k < 0 || k > F) {
      if (f == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
      k = k < 0 ? 0 : F;
    }
  }
  uint32_t key = 0;
  if (dyn && f < F) {
    key = ordered_key(seg_score[int64_t(lh) * F + f]);
    keys[f] = key;
  }
  __syncthreads();
  bool keep = false;
  if (f < F) {
    if (dyn) {
      int rank = 0;
      for (int g = 0; g < F; ++g) {
        const uint32_t kg = keys[g];
        rank += (kg > key) || (kg == key && g < f);
      }
      keep = rank < k;
    } else {
      keep = static_mask[int64_t(lh) * F + f] != 0;
    }
  }
  const unsigned ballot = __ballot_sync(0xffffffffu, keep);
  const int lane = f & 31, warp = f >> 5;
  if (lane == 0) warp_counts[warp] = __popc(ballot);
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_counts[w];
  if (keep) kept_idx[int64_t(lh) * F + base + __popc(ballot & ((1u << lane) - 1u))] = f;
  if (f == 0) {
    int total = 0;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) total += warp_counts[w];
    kept_cnt[lh] = total;
  }
}

cudaError_t launch_select_frame(const Dims& d, const float* seg_score, const uint8_t* head_role,
                                const uint8_t* static_mask, const int32_t* k_per_head,
                                int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                cudaStream_t s) {
  const int threads = d.F <= 32 ? 32 : ((d.F + 31) / 32) * 32;
  return launch_kernel(select_frame_kernel, dim3(d.LH), dim3(threads),
                       sizeof(uint32_t) * (d.F > 0 ? d.F : 1), s, d.pdl, d.F, seg_score, head_role,
                       static_mask, k_per_head, kept_idx, kept_cnt, status);
}

// ---------------------------------------------------------------------------

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelBatch = 8;  // key loads in flight per thread

// Keys cached in shared memory when they fit (the 14B workload's 18720
// candidates take 73 KB); otherwise every pass re-reads them (from L2).
constexpr int64_t kSelCacheKeys = 40960;
// With at most kSelCandMaxKeys cached keys, the keys that survive the first
// pass (those in the threshold's top-byte bin) are also copied to a list of
// up to kSelCandKeys entries, and the later passes scan only that list.
constexpr int64_t kSelCandMaxKeys = 24576;
constexpr int64_t kSelCandKeys = 16384;

__global__ void __launch_bounds__(kSelThreads)
select_token_kernel(int64_t n_c, int64_t S, int64_t R, int64_t N, int cached, int cand_cap,
                    const float* __restrict__ phi, const int32_t* __restrict__ k_per_head,
                    int32_t* __restrict__ kept_idx, int32_t* __restrict__ kept_cnt,
                    int32_t* status) {
  extern __shared__ uint32_t skeys[];  // [n_c] keys if cached, then [cand_cap] candidates
  uint32_t* cand = skeys + (cached ? n_c : 0);
  __shared__ unsigned hist[256];
  __shared__ unsigned whist[kSelWarps][256];  // one histogram per warp
  __shared__ int warp_gt[kSelWarps], warp_eq[kSelWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int64_t s_need;
  __shared__ int s_cand_n;
  pdl_wait();
  const int lh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* ph = phi + int64_t(lh) * n_c;
  int32_t* out = kept_idx + int64_t(lh) * N;
  int64_t C = k_per_head[lh];
  if (C < 0 || C > n_c) {
    if (tid == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
    C = C < 0 ? 0 : n_c;
  }
  for (int64_t i = tid; i < S; i += kSelThreads) out[i] = int32_t(i);
  for (int64_t i = tid; i < R; i += kSelThreads) out[S + C + i] = int32_t(N - R + i);
  if (tid == 0) kept_cnt[lh] = int32_t(S + C + R);
  if (C == 0) return;
  if (cached) {
    // kSelBatch independent loads in flight per thread before any is stored
    for (int64_t j0 = tid; j0 < n_c; j0 += int64_t(kSelThreads) * kSelBatch) {
      float v[kSelBatch];
#pragma unroll
      for (int u = 0; u < kSelBatch; ++u) {
        const int64_t j = j0 + int64_t(u) * kSelThreads;
        v[u] = j < n_c ? __ldcs(ph + j) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kSelBatch; ++u) {
        const int64_t j = j0 + int64_t(u) * kSelThreads;
        if (j < n_c) skeys[j] = ordered_key(v[u]);
      }
    }
    __syncthreads();
  }
  auto key_at = [&](int64_t j) -> uint32_t { return cached ? skeys[j] : ordered_key(ph[j]); };

  // Radix select of the C-th largest key, most significant byte first.  Each
  // warp counts into a histogram of its own (lanes that hit the same bin are
  // merged by __match_any_sync into one shared-memory add), so the many keys
  // that share a bin -- scores of one magnitude share their top byte -- never
  // contend across warps; the 32 histograms are then summed per bin in warp
  // order.
  uint32_t prefix = 0, pmask = 0;
  int64_t need = C;
  int64_t list_n = -1;  // after the first pass: the candidate list's length, or -1 (scan all)
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = lane; b < 256; b += 32) whist[warp][b] = 0;
    __syncwarp();
    const int64_t n_scan = list_n < 0 ? n_c : list_n;
    for (int64_t base = int64_t(warp) * 32; base < n_scan; base += kSelThreads) {
      const int64_t j = base + lane;
      uint32_t bin = 256;  // no bin
      if (j < n_scan) {
        const uint32_t key = list_n < 0 ? key_at(j) : cand[j];
        if ((key & pmask) == prefix) bin = (key >> shift) & 255u;
      }
      const unsigned grp = __match_any_sync(0xffffffffu, bin);
      if (bin < 256 && lane == __ffs(grp) - 1) whist[warp][bin] += unsigned(__popc(grp));
      __syncwarp();
    }
    __syncthreads();
    if (tid < 256) {
      unsigned c = 0;
#pragma unroll 8
      for (int w = 0; w < kSelWarps; ++w) c += whist[w][tid];
      hist[tid] = c;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l owns bins 8*(31-l) .. 8*(31-l)+7 (lane 0 the highest); a warp
      // inclusive scan from the top finds the bin where the count of larger
      // keys first reaches `need`.
      const int b0 = 8 * (31 - lane);
      unsigned cnt = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) cnt += hist[b0 + k];
      unsigned incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const unsigned excl = incl - cnt;
      const bool here = int64_t(excl) < need && int64_t(incl) >= need;
      const unsigned who = __ballot_sync(0xffffffffu, here);
      if (lane == __ffs(who) - 1) {
        int64_t above = excl;
        int b = b0 + 7;
        for (; b > b0; --b) {
          if (above + int64_t(hist[b]) >= need) break;
          above += hist[b];
        }
        s_prefix = prefix | (uint32_t(b) << shift);
        s_need = need - above;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    pmask |= 255u << shift;
    if (pass == 0 && cand_cap > 0) {
      // the keys left in the running (top byte = the threshold's) as a list
      if (tid == 0) s_cand_n = 0;
      __syncthreads();
      for (int64_t base = int64_t(warp) * 32; base < n_c; base += kSelThreads) {
        const int64_t j = base + lane;
        const uint32_t key = j < n_c ? key_at(j) : 0u;
        const bool hit = j < n_c && (key & pmask) == prefix;
        const unsigned bh = __ballot_sync(0xffffffffu, hit);
        int at = 0;
        if (lane == 0 && bh) at = atomicAdd(&s_cand_n, __popc(bh));
        at = __shfl_sync(0xffffffffu, at, 0) + __popc(bh & ((1u << lane) - 1u));
        if (hit && at < cand_cap) cand[at] = key;
      }
      __syncthreads();
      if (s_cand_n <= cand_cap) list_n = s_cand_n;  // else every pass scans all keys
    }
    __syncthreads();
  }
  const uint32_t t = prefix;  // exact key of the C-th largest score
  // Stable compaction in index order: every key > t, and the first `need`
  // keys == t.  Before position j, gt_before keys > t and eq_before keys == t
  // occur, of which min(eq_before, need) are taken.  Warp w owns the
  // contiguous keys [w0, w1): a first sweep counts its (gt, eq) keys, one
  // block scan gives every warp its counts before w0, a second sweep writes.
  const int64_t per_warp = ((n_c + kSelWarps - 1) / kSelWarps + 31) / 32 * 32;
  const int64_t w0 = int64_t(warp) * per_warp;
  const int64_t w1 = w0 + per_warp < n_c ? w0 + per_warp : n_c;
  int gt_w = 0, eq_w = 0;
  for (int64_t j0 = w0; j0 < w1; j0 += 32) {
    const int64_t j = j0 + lane;
    const uint32_t key = j < w1 ? key_at(j) : 0u;
    gt_w += __popc(__ballot_sync(0xffffffffu, j < w1 && key > t));
    eq_w += __popc(__ballot_sync(0xffffffffu, j < w1 && key == t));
  }
  if (lane == 0) {
    warp_gt[warp] = gt_w;
    warp_eq[warp] = eq_w;
  }
  __syncthreads();
  if (warp == 0) {  // exclusive prefixes of the per-warp counts, in warp order
    const int g = warp_gt[lane], e = warp_eq[lane];
    int ig = g, ie = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int vg = __shfl_up_sync(0xffffffffu, ig, o), ve = __shfl_up_sync(0xffffffffu, ie, o);
      if (lane >= o) {
        ig += vg;
        ie += ve;
      }
    }
    __syncwarp();
    warp_gt[lane] = ig - g;
    warp_eq[lane] = ie - e;
  }
  __syncthreads();
  int64_t gt_seen = warp_gt[warp], eq_seen = warp_eq[warp];
  const unsigned below = (1u << lane) - 1u;
  for (int64_t j0 = w0; j0 < w1; j0 += 32) {
    const int64_t j = j0 + lane;
    const uint32_t key = j < w1 ? key_at(j) : 0u;
    const bool gt = j < w1 && key > t;
    const bool eq = j < w1 && key == t;
    const unsigned bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
    const int64_t gt_before = gt_seen + __popc(bg & below);
    const int64_t eq_before = eq_seen + __popc(be & below);
    if (gt || (eq && eq_before < need)) {
      const int64_t pos = gt_before + (eq_before < need ? eq_before : need);
      out[S + pos] = int32_t(S + j);
    }
    gt_seen += __popc(bg);
    eq_seen += __popc(be);
  }
}

// Frame mode with per-token static masks: kept lists in tokens.  Dynamic
// heads rank their frames as above, then write the tokens of the kept frames
// in order; static heads compact the ascending tokens of their mask (block
// scan per 1024 tokens).  One 1024-thread CTA per (layer, head).
__global__ void __launch_bounds__(kSelThreads)
select_frame_tokens_kernel(int F, int T, int64_t N, const float* __restrict__ seg_score,
                           const uint8_t* __restrict__ head_role,
                           const uint8_t* __restrict__ static_mask,
                           const int32_t* __restrict__ k_per_head, int32_t* __restrict__ kept_idx,
                           int32_t* __restrict__ kept_cnt, int32_t* status) {
  __shared__ uint32_t keys[1024];
  __shared__ int32_t kf[1024];
  __shared__ int warp_tot[kSelWarps];
  __shared__ int s_cnt;
  pdl_wait();
  const int lh = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int32_t* out = kept_idx + int64_t(lh) * N;
  if (head_role[lh]) {
    int k = k_per_head[lh];
    if (k < 0 || k > F) {
      if (tid == 0) report(status, FKV_ERR_DEVICE_ARG, lh);
      k = k < 0 ? 0 : F;
    }
    uint32_t key = 0;
    if (tid < F) keys[tid] = key = ordered_key(seg_score[int64_t(lh) * F + tid]);
    __syncthreads();
    bool keep = false;
    if (tid < F) {
      int rank = 0;
      for (int g = 0; g < F; ++g) {
        const uint32_t kg = keys[g];
        rank += (kg > key) || (kg == key && g < tid);
      }
      keep = rank < k;
    }
    // ascending kept frames
    const unsigned b = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_tot[warp] = __popc(b);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    if (keep) kf[before + __popc(b & ((1u << lane) - 1u))] = tid;
    __syncthreads();
    const int64_t n_out = int64_t(total) * T;
    for (int64_t o = tid; o < n_out; o += kSelThreads) {
      const int64_t pfr = o / T;
      out[o] = int32_t(int64_t(kf[pfr]) * T + (o - pfr * T));
    }
    if (tid == 0) kept_cnt[lh] = int32_t(n_out);
    return;
  }
  // static head: tokens of the mask, ascending
  const uint8_t* mk = static_mask + int64_t(lh) * N;
  int64_t base = 0;
  for (int64_t c0 = 0; c0 < N; c0 += kSelThreads) {
    const int64_t j = c0 + tid;
    const bool keep = j < N && mk[j] != 0;
    const unsigned b = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) warp_tot[warp] = __popc(b);
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < kSelWarps; ++w) {
      before += w < warp ? warp_tot[w] : 0;
      total += warp_tot[w];
    }
    __syncthreads();
    if (keep) out[base + before + __popc(b & ((1u << lane) - 1u))] = int32_t(j);
    base += total;
  }
  if (tid == 0) s_cnt = int(base);
  __syncthreads();
  if (tid == 0) kept_cnt[lh] = s_cnt;
}

cudaError_t launch_select_frame_tokens(const Dims& d, const float* seg_score,
                                       const uint8_t* head_role, const uint8_t* static_mask,
                                       const int32_t* k_per_head, int32_t* kept_idx,
                                       int32_t* kept_cnt, int32_t* status, cudaStream_t s) {
  return launch_kernel(select_frame_tokens_kernel, dim3(d.LH), dim3(kSelThreads), 0, s, d.pdl,
                       d.F, d.T, d.N, seg_score, head_role, static_mask, k_per_head, kept_idx,
                       kept_cnt, status);
}

cudaError_t launch_select_token(const Dims& d, const float* seg_score, const int32_t* k_per_head,
                                int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                cudaStream_t s) {
  const int cached = d.nseg <= kSelCacheKeys;
  const int cand_cap = d.nseg <= kSelCandMaxKeys ? int(kSelCandKeys) : 0;
  const size_t smem = sizeof(uint32_t) * ((cached ? size_t(d.nseg) : 0) + size_t(cand_cap) + 1);
  static_assert(kSelCandMaxKeys + kSelCandKeys <= kSelCacheKeys, "dynamic shared memory bound");
  cudaError_t e = cudaFuncSetAttribute(select_token_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(sizeof(uint32_t) * (kSelCacheKeys + 1)));
  if (e != cudaSuccess) return e;
  return launch_kernel(select_token_kernel, dim3(d.LH), dim3(kSelThreads), smem, s, d.pdl,
                       d.nseg, d.S, d.R, d.N, cached, cand_cap, seg_score, k_per_head, kept_idx,
                       kept_cnt, status);
}

}  // namespace fkv
