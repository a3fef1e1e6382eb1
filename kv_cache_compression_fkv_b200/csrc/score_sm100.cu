// Step 2 on the tensor cores: per-frame softmax statistics of the dynamic
// heads' scoring queries (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
// "关键模块" 3: history grouped by frame, each group scored by the current
// queries' attention).
//
// A CTA owns (layer*head, 128 scoring queries, one half of a history frame):
// the frame's T keys are cut into 128-key blocks that start at the frame's
// first token, and the blocks are split into kScoreSplit sub-segments of
// consecutive blocks, so equal frames are reduced in exactly the same order
// (bit-equal statistics) while the grid has kScoreSplit times as many,
// shorter CTAs.  For each query row i the CTA produces the sub-segment max
// m_{g,i} and sum l_{g,i} = sum_{j in g} 2^(z_ij - m_{g,i}) of the base-2
// logits z = scale*log2(e)*q.k; score_finalize_kernel merges them per row and
// sums the frame masses in a fixed order.
//
// Warp roles (320 threads): warps 0-7 fold the logit tiles into (m, l), two
// threads per query row (TMEM lane) with 64 columns each, merged at the end;
// warp 8 issues the TMA loads (Q tile once; K blocks into a 2-stage ring,
// 128-byte swizzle; the scoring rows q_cur[i*stride] come from a strided
// tensor map); warp 9 issues S = Q K^T into a TMEM double buffer, so the MMAs
// of the next block overlap the statistics of the current one.  96 KB of
// shared memory and 256 TMEM columns let two CTAs share an SM.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {

constexpr int kScoreStages = 2;
constexpr int kScoreThreads = 320;
constexpr int kScoreStatThreads = 256;
constexpr int kScoreProducerWarp = 8;
constexpr int kScoreMmaWarp = 9;
constexpr uint32_t kScoreIdesc = idesc_bf16(128, 128, false);
constexpr uint32_t kSOffQ = 0;
constexpr uint32_t kSOffK = kTileBytes;
constexpr uint32_t kSOffBar = kSOffK + kScoreStages * kTileBytes;

struct ScoreBars {
  uint64_t q_full;
  uint64_t k_full[kScoreStages], k_empty[kScoreStages];
  uint64_t s_full[2], s_free[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  float2 xml[2][128];  // [column half][row] partial (max, sum) for the end merge
};

constexpr size_t kScoreSmem = kSOffBar + sizeof(ScoreBars) + 1024;

struct ScoreArgs {
  int T, G, E;  // tokens per frame; history sub-segments (F * kScoreSplit); entries per head
  int Lq, with_chunk;
  int64_t n_s;
  float sl2;
  const uint8_t* head_role;
  float2* part_ml;
  int32_t* status;
};

__device__ __forceinline__ bool warp_wait_s(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ void drain_wait_s(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
}

// (m, l) of the union of two partial softmax sums; empty parts are (-inf, 0).
__device__ __forceinline__ float2 merge_ml(float2 a, float2 b) {
  const float M = fmaxf(a.x, b.x);
  if (M == -INFINITY) return make_float2(-INFINITY, 0.f);
  return make_float2(M, a.y * ex2(a.x - M) + b.y * ex2(b.x - M));
}

__global__ void __launch_bounds__(kScoreThreads, 2)
score_sm100_kernel(const __grid_constant__ CUtensorMap tm_qs,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_kc, const ScoreArgs a) {
  const int qt = blockIdx.x, g = blockIdx.y, lh = blockIdx.z;
  if (!a.head_role[lh]) return;  // static head: nothing to score (uniform per CTA)
  // Key range of this CTA: a history sub-segment, or (last entry) the chunk's
  // own keys when they join the normaliser.
  const bool chunk = g >= a.G;
  const CUtensorMap* tmk = chunk ? &tm_kc : &tm_k;
  int row0, nkeys;
  if (chunk) {
    row0 = 0;
    nkeys = a.Lq;
  } else {
    // sub-segment `sub` of frame f: its blocks [bs, be) of the frame's nbf,
    // bs = ceil(sub * nbf / split) (equal frames are cut at the same blocks)
    const int f = g / kScoreSplit, sub = g - f * kScoreSplit;
    const int nbf = (a.T + 127) / 128;
    const int bs = (sub * nbf + kScoreSplit - 1) / kScoreSplit;
    const int be = ((sub + 1) * nbf + kScoreSplit - 1) / kScoreSplit;
    row0 = f * a.T + bs * 128;
    nkeys = (be * 128 < a.T ? be * 128 : a.T) - bs * 128;
  }
  const int b0 = 0, b1 = nkeys > 0 ? (nkeys + 127) / 128 : 0;
  float2* out = a.part_ml + (int64_t(lh) * a.E + g) * a.n_s;
  if (b0 >= b1) {  // empty sub-segment (a frame of one block): neutral statistics
    const int64_t i = int64_t(qt) * 128 + threadIdx.x;
    if (threadIdx.x < 128 && i < a.n_s) out[i] = make_float2(-INFINITY, 0.f);
    return;
  }
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  ScoreBars* bars = reinterpret_cast<ScoreBars*>(sm + kSOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], kScoreStatThreads);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kScoreMmaWarp) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int row = (warp & 3) * 32 + lane, half = warp >> 2;
  float m = -INFINITY, l = 0.f;

  if (warp == kScoreProducerWarp) {
    if (lane == 0) {
      prefetch_tmap(&tm_qs);
      prefetch_tmap(tmk);
      mbar_expect_tx(&bars->q_full, kTileBytes);
      tma_load_tile(sm + kSOffQ, &tm_qs, &bars->q_full, qt * 128, lh);
      uint32_t issued = 0;
      for (int b = b0; b < b1; ++b, ++issued) {
        const uint32_t s = issued % kScoreStages, u = issued / kScoreStages;
        if (!mbar_wait(&bars->k_empty[s], (u & 1) ^ 1, abort)) break;
        mbar_expect_tx(&bars->k_full[s], kTileBytes);
        tma_load_tile(sm + kSOffK + s * kTileBytes, tmk, &bars->k_full[s], row0 + b * 128, lh);
      }
      for (uint32_t i = issued > kScoreStages ? issued - kScoreStages : 0; i < issued; ++i)
        drain_wait_s(&bars->k_full[i % kScoreStages], (i / kScoreStages) & 1);
      drain_wait_s(&bars->q_full, 0);
    }
  } else if (warp == kScoreMmaWarp) {
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      const uint32_t qbase = smem_u32(sm + kSOffQ);
      for (uint32_t it = 0; ok && it < uint32_t(b1 - b0); ++it) {
        const uint32_t s = it % kScoreStages, u = it / kScoreStages;
        const uint32_t sb = it & 1, su = it >> 1;
        if (!(ok = mbar_wait(&bars->k_full[s], u & 1, abort))) break;
        if (!(ok = mbar_wait(&bars->s_free[sb], (su & 1) ^ 1, abort))) break;
        tc_fence_after();
        const uint32_t kbase = smem_u32(sm + kSOffK + s * kTileBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + sb * 128, kmajor_desc(qbase, k), kmajor_desc(kbase, k), kScoreIdesc,
                 k > 0 ? 1u : 0u);
        mma_commit(&bars->s_full[sb]);
        mma_commit(&bars->k_empty[s]);
      }
      mma_commit(&bars->mma_done);
      drain_wait_s(&bars->mma_done, 0);
    }
  } else {
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const float2 sl2x2 = make_float2(a.sl2, a.sl2);
    bool ok = true;
    for (uint32_t it = 0; ok && it < uint32_t(b1 - b0); ++it) {
      const uint32_t sb = it & 1, su = it >> 1;
      const int cols_left = nkeys - int(it) * 128 - 64 * half;
      const int nv = cols_left < 0 ? 0 : (cols_left < 64 ? cols_left : 64);
      if (!(ok = warp_wait_s(&bars->s_full[sb], su & 1, abort))) break;
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tmem + lane_addr + sb * 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tmem + lane_addr + sb * 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[sb]);
      if (nv < 64) {  // columns past the frame's last token never count
#pragma unroll
        for (int i = 0; i < 64; ++i)
          if (i >= nv) r[i] = 0xff800000u;  // -inf
      }
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(__uint_as_float(r[k]), __uint_as_float(r[k + 8]));
#pragma unroll
      for (int i = 16; i < 64; i += 16)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mx[k] = fmax3(mx[k], __uint_as_float(r[i + k]), __uint_as_float(r[i + k + 8]));
      const float bmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                               fmaxf(mx[6], mx[7]));
      const float m_new = fmaxf(m, bmax * a.sl2);  // scale > 0
      const float mref = m_new == -INFINITY ? 0.f : m_new;
      const float2 negm2 = make_float2(-mref, -mref);
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 e = ffma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                               sl2x2, negm2);
        acc[i & 3] = fadd2(acc[i & 3], make_float2(ex2(e.x), ex2(e.y)));
      }
      const float2 s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      l = (m == -INFINITY ? 0.f : l * ex2(m - mref)) + (s2.x + s2.y);
      m = m_new;
    }
    bars->xml[half][row] = make_float2(m, l);
  }

  __syncthreads();
  if (warp < 4 && !*abort) {
    const int64_t i = int64_t(qt) * 128 + row;
    if (i < a.n_s) out[i] = merge_ml(bars->xml[0][row], bars->xml[1][row]);
  }
  if (warp == kScoreMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && *abort) report(a.status, FKV_ERR_TIMEOUT, lh);
}

}  // namespace sm100

cudaError_t launch_score_frame_sm100(const Dims& d, const void* q_cur, const void* k_hist,
                                     const void* k_cur, const uint8_t* head_role, float2* part_ml,
                                     int32_t* status, cudaStream_t s) {
  using namespace sm100;
  const uint64_t row_b = 128 * 2;
  CUtensorMap tqs, tk, tkc;
  if (!make_tmap_bf16(&tqs, q_cur, d.n_s, d.LH, row_b * d.stride, d.Lq * row_b) ||
      !make_tmap_bf16(&tk, k_hist, d.N, d.LH, row_b, d.N * row_b))
    return cudaErrorInvalidValue;
  if (d.score_with_chunk) {
    if (!make_tmap_bf16(&tkc, k_cur, d.Lq, d.LH, row_b, d.Lq * row_b)) return cudaErrorInvalidValue;
  } else {
    tkc = tk;  // never read
  }
  ScoreArgs a;
  a.T = d.T;
  a.G = d.F * kScoreSplit;
  a.E = a.G + 1;
  a.Lq = int(d.Lq);
  a.with_chunk = d.score_with_chunk ? 1 : 0;
  a.n_s = d.n_s;
  a.sl2 = d.scale * 1.4426950408889634f;
  a.head_role = head_role;
  a.part_ml = part_ml;
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(score_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kScoreSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned((d.n_s + 127) / 128), unsigned(a.G + a.with_chunk), unsigned(d.LH));
  score_sm100_kernel<<<grid, kScoreThreads, kScoreSmem, s>>>(tqs, tk, tkc, a);
  return cudaGetLastError();
}

}  // namespace fkv
