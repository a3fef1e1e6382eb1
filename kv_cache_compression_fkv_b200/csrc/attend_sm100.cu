// Step 5 on the tensor cores: the chunk's queries attend to the compressed
// history followed by the chunk's own keys (Forcing-KV,
// ai-feeds.com/i/paper/2605.09681, "输出与工程收益": the compressed KV
// replaces the cache inside attention; "与现有产品/工作流的接口" step 2).
//
// out_i = sum_j softmax_j(scale * q_i . k_j) v_j over keys = k_comp rows
// [0, kept rows) then k_cur rows [0, Lq), no causal mask; bf16 in, fp32
// accumulation, bf16 out.
//
// One persistent CTA per SM walks (layer*head, 128-query tile) work items.
// Warp roles (320 threads):
//   warps 0-7  softmax: query row r = 32*(w%4) + lane (= TMEM lane r) is
//              shared by warps w and w+4, each owning 64 of the tile's 128
//              key columns; the two exchange their partial row max through
//              shared memory, synchronised by a 64-arrival mbarrier per pair
//              (bounded waits, so an aborting partner cannot hang the other).  They read the fp32
//              logits S from TMEM, keep the running row max m (and a partial
//              row sum l each), write P = 2^(S*scale*log2e - m) as bf16 into
//              TMEM, and rescale the fp32 O accumulator in TMEM only when m
//              grows by more than 2^8 (lazy rescaling: P stays <= 256, exact
//              after the final 1/l).  Epilogue: O / l -> bf16 -> global.
//   warp 8     TMA producer: the Q tile once per work item, then K and V
//              tiles of 128 keys into a 3-stage ring (128-byte swizzle).
//   warp 9     MMA issuer (one thread) and TMEM owner: S = Q K^T with both
//              operands in shared memory, O += P V with P read from TMEM and
//              V (MN-major) from shared memory.
// TMEM (512 columns): S double buffer [0,256), O [256,384), P double buffer
// [384,512) (bf16 pairs).  The MMA of S_{j+1} overlaps the softmax of block j,
// and O += P_{j-1} V_{j-1} overlaps it as well.
//
// Key tiles past the valid rows of a range are masked (logit -> -inf) and
// their V rows zeroed in shared memory before use, so compressed-cache rows
// past the kept count are never read as data, whatever they hold.  Every
// mbarrier wait is bounded; on timeout the CTA records FKV_ERR_TIMEOUT, waits
// (bounded) for its own copies and MMAs, frees TMEM and returns.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {
namespace sm100 {

constexpr int kKVStages = 3;
constexpr int kAttnThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColP = 384;
constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 128, true);
constexpr float kRescaleLog2 = 8.0f;

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTileBytes;
constexpr uint32_t kOffV = kOffK + kKVStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kKVStages * kTileBytes;

struct AttnBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKVStages], k_empty[kKVStages];
  uint64_t v_full[kKVStages], v_empty[kKVStages];
  uint64_t s_full[2], s_free[2], p_full[2], pv_done[2];
  uint64_t o_free, mma_done;
  uint32_t tmem_base;
  int abort;
  uint64_t xbar[2][4];      // [round parity][row quarter]: 64 arrivals (warps w, w+4)
  float xval[2][2][128];    // [round parity][column half][row] partial row max / sum
};

// No alignment slack fits under the 227 KB limit: the kernel checks that the
// dynamic shared memory base is 1024-byte aligned and reports an error if not.
constexpr size_t kAttnSmem = kOffBar + sizeof(AttnBars);
static_assert(kAttnSmem <= 232448, "attention shared memory above the per-CTA limit");

struct AttnArgs {
  int64_t Lq, comp_rows, seg_len, max_kept;
  int n_qtiles, n_tiles;
  float sl2;
  const int32_t* kept_cnt;
  __nv_bfloat16* out;
  int32_t* status;
};

struct Tile {
  int lh, qt, nbA, nb;
  int64_t nA;
};

__device__ __forceinline__ Tile decode(const AttnArgs& a, int tile) {
  Tile t;
  t.lh = tile / a.n_qtiles;
  t.qt = tile - t.lh * a.n_qtiles;
  int64_t cnt = a.kept_cnt[t.lh];
  cnt = cnt < 0 ? 0 : (cnt > a.max_kept ? a.max_kept : cnt);
  int64_t nA = cnt * a.seg_len;
  if (nA > a.comp_rows) nA = a.comp_rows;
  t.nA = nA;
  t.nbA = int((nA + 127) / 128);
  t.nb = t.nbA + int((a.Lq + 127) / 128);
  return t;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// Bounded wait that ignores the abort flag: used to let this CTA's own
// copies and MMAs finish before its shared memory and TMEM are released.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return;
}


__global__ void __launch_bounds__(kAttnThreads, 1)
attend_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {  // uniform: every thread sees the same base
    if (threadIdx.x == 0) report(a.status, FKV_ERR_UNSUPPORTED, blockIdx.x);
    return;
  }
  uint8_t* sm = smem_raw;
  AttnBars* bars = reinterpret_cast<AttnBars*>(sm + kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kKVStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->s_free[b], kSoftmaxThreads);
      mbar_init(&bars->p_full[b], kSoftmaxThreads);
      mbar_init(&bars->pv_done[b], 1);
    }
    mbar_init(&bars->o_free, kSoftmaxThreads);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bars->xbar[0][q], 64);
      mbar_init(&bars->xbar[1][q], 64);
    }
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_vc);
      prefetch_tmap(&tm_kn);
      prefetch_tmap(&tm_vn);
      uint32_t it_k = 0, it_v = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const Tile t = decode(a, tile);
        if (!(ok = mbar_wait(&bars->q_empty, (tc & 1) ^ 1, abort))) break;
        mbar_expect_tx(&bars->q_full, kTileBytes);
        tma_load_tile(sm + kOffQ, &tm_q, &bars->q_full, t.qt * 128, t.lh);
        ++tc;
        for (int j = 0; j < t.nb; ++j) {
          const bool inA = j < t.nbA;
          const int row = (inA ? j : j - t.nbA) * 128;
          const uint32_t s = it_k % kKVStages, u = it_k / kKVStages;
          if (!(ok = mbar_wait(&bars->k_empty[s], (u & 1) ^ 1, abort))) break;
          mbar_expect_tx(&bars->k_full[s], kTileBytes);
          tma_load_tile(sm + kOffK + s * kTileBytes, inA ? &tm_kc : &tm_kn, &bars->k_full[s], row,
                        t.lh);
          ++it_k;
          if (!(ok = mbar_wait(&bars->v_empty[s], (u & 1) ^ 1, abort))) break;
          mbar_expect_tx(&bars->v_full[s], kTileBytes);
          tma_load_tile(sm + kOffV + s * kTileBytes, inA ? &tm_vc : &tm_vn, &bars->v_full[s], row,
                        t.lh);
          ++it_v;
        }
      }
      // Let every copy this thread issued land before the CTA exits.
      for (uint32_t i = it_k > kKVStages ? it_k - kKVStages : 0; i < it_k; ++i)
        drain_wait(&bars->k_full[i % kKVStages], (i / kKVStages) & 1);
      for (uint32_t i = it_v > kKVStages ? it_v - kKVStages : 0; i < it_v; ++i)
        drain_wait(&bars->v_full[i % kKVStages], (i / kKVStages) & 1);
      if (tc > 0) drain_wait(&bars->q_full, (tc - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t it = 0, tc = 0;
      bool ok = true, pend = false, p_first = false;
      uint32_t p_it = 0, p_tc = 0;
      auto issue_pv = [&]() -> bool {
        const uint32_t pb = p_it & 1, pu = p_it >> 1;
        const uint32_t s = p_it % kKVStages, u = p_it / kKVStages;
        if (p_first && !mbar_wait(&bars->o_free, (p_tc & 1) ^ 1, abort)) return false;
        if (!mbar_wait(&bars->p_full[pb], pu & 1, abort)) return false;
        if (!mbar_wait(&bars->v_full[s], u & 1, abort)) return false;
        tc_fence_after();
        const uint32_t vbase = smem_u32(sm + kOffV + s * kTileBytes);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tmem + kColO, tmem + kColP + pb * 64 + k * 8, mnmajor_desc(vbase, k), kIdescPV,
                 (p_first && k == 0) ? 0u : 1u);
        mma_commit(&bars->pv_done[pb]);
        mma_commit(&bars->v_empty[s]);
        return true;
      };
      const uint32_t qbase = smem_u32(sm + kOffQ);
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++tc) {
        const Tile t = decode(a, tile);
        if (!(ok = mbar_wait(&bars->q_full, tc & 1, abort))) break;
        tc_fence_after();
        for (int j = 0; j < t.nb; ++j, ++it) {
          const uint32_t sb = it & 1, su = it >> 1;
          const uint32_t s = it % kKVStages, u = it / kKVStages;
          if (!(ok = mbar_wait(&bars->k_full[s], u & 1, abort))) break;
          if (!(ok = mbar_wait(&bars->s_free[sb], (su & 1) ^ 1, abort))) break;
          tc_fence_after();
          const uint32_t kbase = smem_u32(sm + kOffK + s * kTileBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + sb * 128, kmajor_desc(qbase, k), kmajor_desc(kbase, k), kIdescQK,
                   k > 0 ? 1u : 0u);
          mma_commit(&bars->s_full[sb]);
          mma_commit(&bars->k_empty[s]);
          if (j == t.nb - 1) mma_commit(&bars->q_empty);
          if (pend && !(ok = issue_pv())) break;
          pend = true;
          p_it = it;
          p_first = j == 0;
          p_tc = tc;
        }
      }
      if (ok && pend) issue_pv();
      // Every MMA issued here completes before TMEM is released.
      mma_commit(&bars->mma_done);
      drain_wait(&bars->mma_done, 0);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int row = (warp & 3) * 32 + lane;
    const int half = warp >> 2;                 // key columns [64*half, 64*half + 64)
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const int quarter = warp & 3;               // rows shared by warps w and w+4
    uint32_t it = 0, xc = 0;
    bool ok = true;
    // Exchange of one float with the partner thread of the same row: round xc
    // uses slot xc & 1; a slot is rewritten only two rounds later, after the
    // partner has arrived on the round in between, i.e. after it read it.
    auto exchange = [&](float v, float* other) -> bool {
      const uint32_t slot = xc & 1;
      bars->xval[slot][half][row] = v;
      mbar_arrive(&bars->xbar[slot][quarter]);
      if (!warp_wait(&bars->xbar[slot][quarter], (xc >> 1) & 1, abort)) return false;
      *other = bars->xval[slot][half ^ 1][row];
      ++xc;
      return true;
    };
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
      const Tile t = decode(a, tile);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < t.nb; ++j, ++it) {
        const uint32_t sb = it & 1, su = it >> 1;
        const bool inA = j < t.nbA;
        const int64_t r0 = int64_t(inA ? j : j - t.nbA) * 128;
        const int64_t rows_left = (inA ? t.nA : a.Lq) - r0;
        const int nv_tile = rows_left < 128 ? int(rows_left) : 128;  // valid keys of the tile
        const int nv = nv_tile - 64 * half < 0 ? 0 : (nv_tile - 64 * half > 64 ? 64 : nv_tile - 64 * half);
        if (!(ok = warp_wait(&bars->s_full[sb], su & 1, abort))) break;
        tc_fence_after();
        uint32_t r[64];
        tmem_ld32(tmem + lane_addr + sb * 128 + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        tmem_ld32(tmem + lane_addr + sb * 128 + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bars->s_free[sb]);
        float sv[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) sv[i] = __uint_as_float(r[i]);
        if (nv < 64) {  // ragged tile: columns past the valid keys never count
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (i >= nv) sv[i] = -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmaxf(sv[k], sv[k + 8]);
#pragma unroll
        for (int i = 16; i < 64; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], sv[i + k], sv[i + k + 8]);
        float pmax = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                           fmaxf(mx8[6], mx8[7]));
        float omax;
        if (!(ok = exchange(pmax, &omax))) break;
        pmax = fmaxf(pmax, omax);
        const float m_new = fmaxf(m, pmax * a.sl2);  // scale > 0
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
          // O holds blocks < j: wait for the last PV, then rescale this half in TMEM.
          const uint32_t pi = it - 1;
          if (!(ok = warp_wait(&bars->pv_done[pi & 1], (pi >> 1) & 1, abort))) break;
          tc_fence_after();
          const float alpha = ex2(m - m_new);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_addr + kColO + half * 64 + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_addr + kColO + half * 64 + c * 32, o);
          }
          tmem_st_wait();
          l *= alpha;
          m = m_new;
        }
        // P_j into TMEM buffer pb once the PV that last read that buffer is done.
        const uint32_t pb = it & 1, pu = it >> 1;
        if (!(ok = warp_wait(&bars->pv_done[pb], (pu & 1) ^ 1, abort))) break;
        tc_fence_after();
        uint32_t pk[32];
        float2 sum4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) sum4[k] = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(a.sl2, a.sl2), negm2 = make_float2(-m, -m);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 e = ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), sl2x2, negm2);
          const float2 p = make_float2(ex2(e.x), ex2(e.y));
          sum4[i & 3] = fadd2(sum4[i & 3], p);
          pk[i] = pack_bf16(p.x, p.y);
        }
        const float2 s2 = fadd2(fadd2(sum4[0], sum4[1]), fadd2(sum4[2], sum4[3]));
        l += s2.x + s2.y;
        tmem_st32(tmem + lane_addr + kColP + pb * 64 + half * 32, pk);
        tmem_st_wait();
        if (nv_tile < 128) {
          // V rows past the valid keys may hold anything (P is 0 there, but
          // 0 * NaN is not 0): zero them before the PV MMA reads the stage.
          const uint32_t s = it % kKVStages, u = it / kKVStages;
          if (!(ok = warp_wait(&bars->v_full[s], u & 1, abort))) break;
          if (row >= nv_tile) {
            uint4* v = reinterpret_cast<uint4*>(sm + kOffV + s * kTileBytes + half * kRegionBytes + row * 128);
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) v[c] = z;
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&bars->p_full[pb]);
      }
      if (!ok) break;
      // Epilogue: O / l -> bf16 -> out, each thread its 64 columns.
      const uint32_t last = it - 1;
      if (!(ok = warp_wait(&bars->pv_done[last & 1], (last >> 1) & 1, abort))) break;
      tc_fence_after();
      uint32_t o[64];
      tmem_ld32(tmem + lane_addr + kColO + half * 64, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
      tmem_ld32(tmem + lane_addr + kColO + half * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      float ol;
      if (!(ok = exchange(l, &ol))) break;
      const float inv = 1.f / (l + ol);
      const int64_t q = int64_t(t.qt) * 128 + row;
      if (q < a.Lq) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + (int64_t(t.lh) * a.Lq + q) * 128 + half * 64);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4 v;
          v.x = pack_bf16(__uint_as_float(o[8 * c + 0]) * inv, __uint_as_float(o[8 * c + 1]) * inv);
          v.y = pack_bf16(__uint_as_float(o[8 * c + 2]) * inv, __uint_as_float(o[8 * c + 3]) * inv);
          v.z = pack_bf16(__uint_as_float(o[8 * c + 4]) * inv, __uint_as_float(o[8 * c + 5]) * inv);
          v.w = pack_bf16(__uint_as_float(o[8 * c + 6]) * inv, __uint_as_float(o[8 * c + 7]) * inv);
          dst[c] = v;
        }
      }
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bars->abort) report(a.status, FKV_ERR_TIMEOUT, blockIdx.x);
}

}  // namespace sm100

int num_sms();

cudaError_t launch_attend_sm100(const Dims& d, const void* q_cur, const void* k_cur,
                                const void* v_cur, const void* k_comp, const void* v_comp,
                                const int32_t* kept_cnt, void* out, int32_t* status,
                                cudaStream_t s) {
  using namespace sm100;
  const uint64_t row_b = 128 * 2;
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  const bool have_comp = d.comp_rows > 0;
  if (!make_tmap_bf16(&tq, q_cur, d.Lq, d.LH, row_b, d.Lq * row_b) ||
      !make_tmap_bf16(&tkn, k_cur, d.Lq, d.LH, row_b, d.Lq * row_b) ||
      !make_tmap_bf16(&tvn, v_cur, d.Lq, d.LH, row_b, d.Lq * row_b))
    return cudaErrorInvalidValue;
  if (have_comp) {
    if (!make_tmap_bf16(&tkc, k_comp, d.comp_rows, d.LH, row_b, d.comp_rows * row_b) ||
        !make_tmap_bf16(&tvc, v_comp, d.comp_rows, d.LH, row_b, d.comp_rows * row_b))
      return cudaErrorInvalidValue;
  } else {  // no compressed rows: never read, any valid map will do
    tkc = tkn;
    tvc = tvn;
  }
  AttnArgs a;
  a.Lq = d.Lq;
  a.comp_rows = d.comp_rows;
  a.seg_len = d.seg_len;
  a.max_kept = d.max_kept;
  a.n_qtiles = int((d.Lq + 127) / 128);
  a.n_tiles = a.n_qtiles * d.LH;
  a.sl2 = d.scale * 1.4426950408889634f;
  a.kept_cnt = kept_cnt;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(attend_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kAttnSmem));
  if (e != cudaSuccess) return e;
  const int grid = a.n_tiles < num_sms() ? a.n_tiles : num_sms();
  attend_sm100_kernel<<<grid, kAttnThreads, kAttnSmem, s>>>(tq, tkc, tvc, tkn, tvn, a);
  return cudaGetLastError();
}

}  // namespace fkv
