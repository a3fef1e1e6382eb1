// Step 2 on the tensor cores: per-block softmax statistics of the dynamic
// heads' scoring queries (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
// "关键模块" 3: history grouped by frame, each group scored by the current
// queries' attention).
//
// Work unit = one 128-key block of one frame (blocks start at the frame's
// first token; the last is ragged) -- or of the chunk's own keys when they join
// the normaliser -- for one dynamic head and one tile of 128 scoring queries.
// For each query row i the unit produces m_{b,i} = max_j z_ij and
// l_{b,i} = sum_j 2^(z_ij - m_{b,i}) over the block's keys j, with base-2
// logits z = scale*log2(e)*q.k, written as entry b of the head's partial
// statistics; the finalize merges the entries per row and sums them per frame
// in a fixed order.  Equal frames are therefore reduced in exactly the same
// order (bit-equal masses) however the units are spread over CTAs.
//
// The grid is persistent (two CTAs per SM by default): the dynamic heads are counted on
// the device and CTA c takes units [c*U/G, (c+1)*U/G) of the U units, ordered
// (dynamic head, query tile, block), so the work is balanced to one block and
// the K pipeline runs on across units.  Warp roles (320 threads): warps 0-7
// fold S into (m, l), two threads per query row (TMEM lane) with 64 columns
// each, merged through a bounded mbarrier exchange; warp 8 issues the TMA
// loads (the query tile when it changes; K blocks into a 2-stage ring, 128-byte
// swizzle; the scoring rows q_cur[i*stride] come from a strided tensor map);
// warp 9 issues S = Q K^T into a TMEM double buffer, so the MMAs of the next
// block overlap the statistics of the current one.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {

// K ring depth and CTAs per SM (shared memory: 32 KB per stage + 32 KB of Q).
#ifndef FKV_SCORE_STAGES
#define FKV_SCORE_STAGES 2
#endif
#ifndef FKV_SCORE_CTAS_PER_SM
#define FKV_SCORE_CTAS_PER_SM 2
#endif
// One exponential pair in FKV_SCORE_POLY_EVERY on the FMA pipe (0: none).
// Measured at 480P / 1080P (30 launches, median): 0 44.0 / 312 us, 8 44.0 /
// 304, 4 42.3 / 304, 2 46.0 / 325.
#ifndef FKV_SCORE_POLY_EVERY
#define FKV_SCORE_POLY_EVERY 4
#endif
constexpr int kScorePolyEvery = FKV_SCORE_POLY_EVERY;
constexpr int kScorePolyDiv = kScorePolyEvery > 0 ? kScorePolyEvery : 1;
static_assert(FKV_POLY_DEG == 3, "scores need the degree-3 exp2 (8.6e-5)");
constexpr int kScoreStages = FKV_SCORE_STAGES;
constexpr int kScoreCtasPerSm = FKV_SCORE_CTAS_PER_SM;
constexpr int kScoreThreads = 320;
constexpr int kScoreHalfThreads = 128;  // one column half of the statistics warps
constexpr int kScoreProducerWarp = 8;
constexpr int kScoreMmaWarp = 9;
constexpr uint32_t kScoreIdesc = idesc_bf16(128, 128, false);
constexpr uint32_t kSOffQ = 0;
constexpr uint32_t kSOffK = kTileBytes;
constexpr uint32_t kSOffBar = kSOffK + kScoreStages * kTileBytes;

struct ScoreBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kScoreStages], k_empty[kScoreStages];
  uint64_t s_full[2], s_free[2];
  uint64_t x_full[2], x_read[2];  // per S buffer: half 1 wrote (m, l) / half 0 read it
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int n_dyn;
  int c_dh, c_lh;      // cursor: dynamic head c_dh is head c_lh (this CTA's first unit)
  float2 xml[2][128];  // [S buffer][row] (m, l) of the second column half
};

constexpr size_t kScoreSmem = kSOffBar + sizeof(ScoreBars) + 1024;

struct ScoreArgs {
  int LH, T, F, nbf, nbc, E;  // blocks per frame / of the chunk (0: chunk not scored)
  int n_qt;
  int Lq;
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

// The d-th dynamic head, scanning on from a cursor (cd, clh) = (index, head)
// of the last one found; -1 when there is none.
__device__ __forceinline__ int dyn_head(const uint8_t* __restrict__ role, int LH, int d, int& cd,
                                        int& clh) {
  if (d < cd) {
    cd = -1;
    clh = -1;
  }
  while (cd < d) {
    ++clh;
    while (clh < LH && !role[clh]) ++clh;
    if (clh >= LH) return -1;
    ++cd;
  }
  return clh;
}

// Walks the units in order: dynamic head dh, query tile qt, block b of that
// (head, tile) = block blk of frame f, or block b - F*nbf of the chunk.  One
// division at the start, counters after.
struct ScoreUnit {
  int dh, qt, b, f, blk;
  int row0;    // first key row of the block in its tensor
  int nk;      // valid keys of the block (1..128)
  bool chunk;  // the block is one of the chunk's own keys

  __device__ __forceinline__ void at(const ScoreArgs& a, int64_t u) {
    const int NB = a.F * a.nbf + a.nbc;
    dh = int(u / (int64_t(a.n_qt) * NB));
    const int rem = int(u - int64_t(dh) * a.n_qt * NB);
    qt = rem / NB;
    b = rem - qt * NB;
    f = b / a.nbf;
    blk = b - f * a.nbf;
    derive(a);
  }
  __device__ __forceinline__ void next(const ScoreArgs& a) {
    ++b;
    if (++blk == a.nbf) {
      blk = 0;
      ++f;
    }
    if (b == a.F * a.nbf + a.nbc) {
      b = f = blk = 0;
      if (++qt == a.n_qt) {
        qt = 0;
        ++dh;
      }
    }
    derive(a);
  }
  __device__ __forceinline__ void derive(const ScoreArgs& a) {
    chunk = f >= a.F;
    if (!chunk) {
      row0 = f * a.T + blk * 128;
      nk = min(128, a.T - blk * 128);
    } else {
      row0 = (b - a.F * a.nbf) * 128;
      nk = min(128, a.Lq - row0);
    }
  }
};

__global__ void __launch_bounds__(kScoreThreads, kScoreCtasPerSm)
score_sm100_kernel(const __grid_constant__ CUtensorMap tm_qs,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_kc, const ScoreArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  ScoreBars* bars = reinterpret_cast<ScoreBars*>(sm + kSOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], 2 * kScoreHalfThreads);
      mbar_init(&bars->x_full[b], kScoreHalfThreads);
      mbar_init(&bars->x_read[b], kScoreHalfThreads);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    bars->n_dyn = 0;
    fence_mbar_init();
  }
  __syncthreads();
  {  // dynamic heads: the units cover only them
    int c = 0;
    for (int i = threadIdx.x; i < a.LH; i += blockDim.x) c += a.head_role[i] != 0;
    if (c) atomicAdd(&bars->n_dyn, c);
  }
  if (warp == kScoreMmaWarp) {
    tmem_alloc(&bars->tmem_base, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int64_t NB = int64_t(a.F) * a.nbf + a.nbc;
  const int64_t U = int64_t(bars->n_dyn) * a.n_qt * NB;
  const int64_t u0 = U * blockIdx.x / gridDim.x, u1 = U * (blockIdx.x + 1) / gridDim.x;
  if (warp == 0) {  // the head of this CTA's first unit, 32 roles per ballot
    int want = u0 < u1 ? int(u0 / (int64_t(a.n_qt) * NB)) : 0, found = -1;
    const int dh0 = want;
    for (int base = 0; base < a.LH && found < 0; base += 32) {
      const int i = base + lane;
      const bool dyn = i < a.LH && a.head_role[i] != 0;
      const unsigned bits = __ballot_sync(0xffffffffu, dyn);
      const int c = __popc(bits);
      if (want < c) {
        const int before = __popc(bits & ((1u << lane) - 1u));
        found = base + __ffs(__ballot_sync(0xffffffffu, dyn && before == want)) - 1;
      } else {
        want -= c;
      }
    }
    if (lane == 0) {
      bars->c_dh = found >= 0 ? dh0 : -1;
      bars->c_lh = found;
    }
  }
  __syncthreads();

  if (warp == kScoreProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_qs);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_kc);
      int cd = bars->c_dh, clh = bars->c_lh, prev = -1;
      uint32_t qn = 0, kn = 0;
      bool ok = true;
      ScoreUnit t;
      if (u0 < u1) t.at(a, u0);
      for (int64_t u = u0; ok && u < u1; ++u, t.next(a)) {
        const int lh = dyn_head(a.head_role, a.LH, t.dh, cd, clh);
        if (lh < 0) break;
        const int key = t.dh * a.n_qt + t.qt;
        if (key != prev) {  // a new query tile once the MMAs on the last one are done
          if (qn > 0 && !(ok = mbar_wait(&bars->q_empty, (qn - 1) & 1, abort))) break;
          mbar_expect_tx(&bars->q_full, kTileBytes);
          tma_load_tile(sm + kSOffQ, &tm_qs, &bars->q_full, t.qt * 128, lh);
          ++qn;
          prev = key;
        }
        const uint32_t s = kn % kScoreStages, use = kn / kScoreStages;
        if (!(ok = mbar_wait(&bars->k_empty[s], (use & 1) ^ 1, abort))) break;
        mbar_expect_tx(&bars->k_full[s], kTileBytes);
        tma_load_tile(sm + kSOffK + s * kTileBytes, t.chunk ? &tm_kc : &tm_k, &bars->k_full[s],
                      t.row0, lh);
        ++kn;
      }
      for (uint32_t i = kn > kScoreStages ? kn - kScoreStages : 0; i < kn; ++i)
        drain_wait_s(&bars->k_full[i % kScoreStages], (i / kScoreStages) & 1);
      if (qn > 0) drain_wait_s(&bars->q_full, (qn - 1) & 1);
    }
  } else if (warp == kScoreMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t qbase = smem_u32(sm + kSOffQ);
      int prev = -1;
      uint32_t qn = 0, it = 0;
      bool ok = true;
      ScoreUnit t;
      if (u0 < u1) t.at(a, u0);
      for (int64_t u = u0; ok && u < u1; ++u, ++it, t.next(a)) {
        const int key = t.dh * a.n_qt + t.qt;
        if (key != prev) {
          if (qn > 0) mma_commit(&bars->q_empty);  // arrives when the last tile's MMAs are done
          if (!(ok = mbar_wait(&bars->q_full, qn & 1, abort))) break;
          ++qn;
          prev = key;
        }
        const uint32_t s = it % kScoreStages, use = it / kScoreStages;
        const uint32_t sb = it & 1, su = it >> 1;
        if (!(ok = mbar_wait(&bars->k_full[s], use & 1, abort))) break;
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
    // ------------------------------------------------------------ statistics warps
    const int row = (warp & 3) * 32 + lane, half = warp >> 2;
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const float2 sl2x2 = make_float2(a.sl2, a.sl2);
    int cd = bars->c_dh, clh = bars->c_lh;
    uint32_t it = 0;
    bool ok = true;
    ScoreUnit t;
    if (u0 < u1) t.at(a, u0);
    for (int64_t u = u0; ok && u < u1; ++u, ++it, t.next(a)) {
      const int lh = dyn_head(a.head_role, a.LH, t.dh, cd, clh);
      const uint32_t sb = it & 1, su = it >> 1;
      const int cols_left = t.nk - 64 * half;
      const int nv = cols_left < 0 ? 0 : (cols_left < 64 ? cols_left : 64);
      if (!(ok = warp_wait_s(&bars->s_full[sb], su & 1, abort))) break;
      tc_fence_after();
      uint32_t r[64];
      tmem_ld32(tmem + lane_addr + sb * 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
      tmem_ld32(tmem + lane_addr + sb * 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->s_free[sb]);
      if (nv < 64) {  // columns past the block's last key never count
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
      const float m = bmax * a.sl2;  // scale > 0; -inf for an empty half
      const float mref = m == -INFINITY ? 0.f : m;
      const float2 negm2 = make_float2(-mref, -mref);
      float2 acc[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float2 e = ffma2(make_float2(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1])),
                               sl2x2, negm2);
        // one pair in FKV_SCORE_POLY_EVERY on the FMA pipe (relative error
        // <= 8.6e-5 per term), the rest on MUFU
        const bool poly = kScorePolyEvery > 0 && i % kScorePolyDiv == kScorePolyDiv - 1;
        acc[i & 3] = fadd2(acc[i & 3], poly ? exp2_poly2(e) : make_float2(ex2(e.x), ex2(e.y)));
      }
      const float2 s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
      const float2 mine = make_float2(m, m == -INFINITY ? 0.f : s2.x + s2.y);
      // merge the two column halves of the row; half 0 writes the entry
      if (half) {
        if (!(ok = warp_wait_s(&bars->x_read[sb], (su & 1) ^ 1, abort))) break;
        bars->xml[sb][row] = mine;
        mbar_arrive(&bars->x_full[sb]);
      } else {
        if (!(ok = warp_wait_s(&bars->x_full[sb], su & 1, abort))) break;
        const float2 other = bars->xml[sb][row];
        mbar_arrive(&bars->x_read[sb]);
        const int64_t i = int64_t(t.qt) * 128 + row;
        if (lh >= 0 && i < a.n_s)
          a.part_ml[(int64_t(lh) * a.n_s + i) * a.E + t.b] = merge_ml(mine, other);
      }
    }
  }

  __syncthreads();
  if (warp == kScoreMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  if (threadIdx.x == 0 && *abort) report(a.status, FKV_ERR_TIMEOUT, blockIdx.x);
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
  const ScoreLayout sl = score_layout(d);
  ScoreArgs a;
  a.LH = d.LH;
  a.T = d.T;
  a.F = d.F;
  a.nbf = sl.split;
  a.nbc = sl.chunk;
  a.E = sl.E;
  a.n_qt = int((d.n_s + 127) / 128);
  a.Lq = int(d.Lq);
  a.n_s = d.n_s;
  a.sl2 = d.scale * 1.4426950408889634f;
  a.head_role = head_role;
  a.part_ml = part_ml;
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(score_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kScoreSmem));
  if (e != cudaSuccess) return e;
  // Persistent: two CTAs per SM, fewer when there are fewer units than that.
  const int64_t units_max = int64_t(d.LH) * a.n_qt * (int64_t(d.F) * a.nbf + a.nbc);
  int64_t grid = int64_t(num_sms()) * kScoreCtasPerSm;
  if (units_max < grid) grid = units_max;
  if (grid < 1) return cudaSuccess;
  score_sm100_kernel<<<unsigned(grid), kScoreThreads, kScoreSmem, s>>>(tqs, tk, tkc, a);
  return cudaGetLastError();
}

}  // namespace fkv
