// Step 2 on the tensor cores: per-frame softmax statistics of the dynamic
// heads' scoring queries (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
// "关键模块" 3: history grouped by frame, each group scored by the current
// queries' attention).
//
// A CTA owns (layer*head, 128 scoring queries, history frame f) and streams
// the frame's T keys in 128-key tiles that start at the frame's first token,
// so every frame is reduced in the same order (equal frames give bit-equal
// statistics).  For each query row i it produces the frame-local max
// m_{f,i} and sum l_{f,i} = sum_{j in f} 2^(z_ij - m_{f,i}) of the base-2
// logits z = scale*log2(e)*q.k; the per-row merge over frames and the
// deterministic sum over rows into the frame mass run afterwards (simt.cu).
//
// Warp roles (192 threads): warps 0-3 hold one query row per thread (TMEM
// lane) and fold each 128x128 fp32 logit tile into (m, l); warp 4 issues
// the TMA loads (Q tile once, K tiles into a 2-stage ring, 128-byte swizzle;
// the scoring rows q_cur[i*stride] come from a strided tensor map); warp 5
// issues S = Q K^T into a TMEM double buffer.  96 KB of shared memory and 256
// TMEM columns let two CTAs share an SM.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {

constexpr int kScoreStages = 2;
constexpr int kScoreThreads = 192;
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
};

constexpr size_t kScoreSmem = kSOffBar + sizeof(ScoreBars) + 1024;

struct ScoreArgs {
  int T, F;
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

__global__ void __launch_bounds__(kScoreThreads, 2)
score_sm100_kernel(const __grid_constant__ CUtensorMap tm_qs,
                   const __grid_constant__ CUtensorMap tm_k, const ScoreArgs a) {
  const int qt = blockIdx.x, f = blockIdx.y, lh = blockIdx.z;
  if (!a.head_role[lh]) return;  // static head: nothing to score (uniform per CTA)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  ScoreBars* bars = reinterpret_cast<ScoreBars*>(sm + kSOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nb = (a.T + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 128);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&tm_qs);
      prefetch_tmap(&tm_k);
      mbar_expect_tx(&bars->q_full, kTileBytes);
      tma_load_tile(sm + kSOffQ, &tm_qs, &bars->q_full, qt * 128, lh);
      uint32_t issued = 0;
      for (int b = 0; b < nb; ++b) {
        const uint32_t s = b % kScoreStages, u = b / kScoreStages;
        if (!mbar_wait(&bars->k_empty[s], (u & 1) ^ 1, abort)) break;
        mbar_expect_tx(&bars->k_full[s], kTileBytes);
        tma_load_tile(sm + kSOffK + s * kTileBytes, &tm_k, &bars->k_full[s], f * a.T + b * 128, lh);
        ++issued;
      }
      for (uint32_t i = issued > kScoreStages ? issued - kScoreStages : 0; i < issued; ++i)
        drain_wait_s(&bars->k_full[i % kScoreStages], (i / kScoreStages) & 1);
      drain_wait_s(&bars->q_full, 0);
    }
  } else if (warp == 5) {
    if (lane == 0) {
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      const uint32_t qbase = smem_u32(sm + kSOffQ);
      for (int b = 0; ok && b < nb; ++b) {
        const uint32_t s = b % kScoreStages, u = b / kScoreStages;
        const uint32_t sb = b & 1, su = b >> 1;
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
    const int row = threadIdx.x;
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int b = 0; b < nb; ++b) {
      const uint32_t sb = b & 1, su = b >> 1;
      const int nv = a.T - b * 128 < 128 ? a.T - b * 128 : 128;
      if (!(ok = warp_wait_s(&bars->s_full[sb], su & 1, abort))) break;
      tc_fence_after();
      uint32_t r[128];
      tmem_ld32(tmem + lane_addr + sb * 128 + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tmem + lane_addr + sb * 128 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld32(tmem + lane_addr + sb * 128 + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
      tmem_ld32(tmem + lane_addr + sb * 128 + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[sb]);
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 128; ++i)
        if (i < nv) mx = fmaxf(mx, __uint_as_float(r[i]) * a.sl2);
      const float m_new = fmaxf(m, mx);
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < 128; ++i)
        if (i < nv) sum += ex2(__uint_as_float(r[i]) * a.sl2 - m_new);
      l = l * ex2(m - m_new) + sum;
      m = m_new;
    }
    const int64_t i = int64_t(qt) * 128 + row;
    if (ok && i < a.n_s) a.part_ml[(int64_t(lh) * a.F + f) * a.n_s + i] = make_float2(m, l);
  }

  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && bars->abort) report(a.status, FKV_ERR_TIMEOUT, lh);
}

}  // namespace sm100

cudaError_t launch_score_frame_sm100(const Dims& d, const void* q_cur, const void* k_hist,
                                     const uint8_t* head_role, float2* part_ml, int32_t* status,
                                     cudaStream_t s) {
  using namespace sm100;
  const uint64_t row_b = 128 * 2;
  CUtensorMap tqs, tk;
  if (!make_tmap_bf16(&tqs, q_cur, d.n_s, d.LH, row_b * d.stride, d.Lq * row_b) ||
      !make_tmap_bf16(&tk, k_hist, d.N, d.LH, row_b, d.N * row_b))
    return cudaErrorInvalidValue;
  ScoreArgs a;
  a.T = d.T;
  a.F = d.F;
  a.n_s = d.n_s;
  a.sl2 = d.scale * 1.4426950408889634f;
  a.head_role = head_role;
  a.part_ml = part_ml;
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(score_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kScoreSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(unsigned((d.n_s + 127) / 128), unsigned(d.F), unsigned(d.LH));
  score_sm100_kernel<<<grid, kScoreThreads, kScoreSmem, s>>>(tqs, tk, a);
  return cudaGetLastError();
}

}  // namespace fkv
