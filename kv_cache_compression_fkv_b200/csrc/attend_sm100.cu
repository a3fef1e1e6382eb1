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
// Warp roles (192 threads):
//   warps 0-3  softmax: thread t owns query row t = TMEM lane t.  Reads the
//              128x128 fp32 logits S from TMEM, keeps a running row max m and
//              sum l, writes P = 2^(S*scale*log2e - m) as bf16 into TMEM, and
//              rescales the fp32 O accumulator in TMEM only when m grows by
//              more than 2^8 (lazy rescaling: P stays <= 256, exact after the
//              final 1/l).  Epilogue: O / l -> bf16 -> global.
//   warp 4     TMA producer: the Q tile once per work item, then K and V
//              tiles of 128 keys into a 3-stage ring (128-byte swizzle).
//   warp 5     MMA issuer (one thread) and TMEM owner: S = Q K^T with both
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
constexpr int kAttnThreads = 192;
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
};

constexpr size_t kAttnSmem = kOffBar + sizeof(AttnBars) + 1024;

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

__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  tmem_ld32(taddr + 0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
  tmem_ld32(taddr + 64, *reinterpret_cast<uint32_t(*)[32]>(&r[64]));
  tmem_ld32(taddr + 96, *reinterpret_cast<uint32_t(*)[32]>(&r[96]));
  tmem_ld_wait();
}

__global__ void __launch_bounds__(kAttnThreads, 1)
attend_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_kc,
                    const __grid_constant__ CUtensorMap tm_vc,
                    const __grid_constant__ CUtensorMap tm_kn,
                    const __grid_constant__ CUtensorMap tm_vn, const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
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
      mbar_init(&bars->s_free[b], 128);
      mbar_init(&bars->p_full[b], 128);
      mbar_init(&bars->pv_done[b], 1);
    }
    mbar_init(&bars->o_free, 128);
    mbar_init(&bars->mma_done, 1);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 4) {
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
  } else if (warp == 5) {
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
    const int row = threadIdx.x;
    const uint32_t lane_addr = uint32_t(warp * 32) << 16;
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
      const Tile t = decode(a, tile);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < t.nb; ++j, ++it) {
        const uint32_t sb = it & 1, su = it >> 1;
        const bool inA = j < t.nbA;
        const int64_t r0 = int64_t(inA ? j : j - t.nbA) * 128;
        const int64_t avail = (inA ? t.nA : a.Lq) - r0;
        const int nv = avail < 128 ? int(avail) : 128;
        if (!(ok = warp_wait(&bars->s_full[sb], su & 1, abort))) break;
        tc_fence_after();
        uint32_t r[128];
        tmem_ld128(tmem + lane_addr + sb * 128, r);
        tc_fence_before();
        mbar_arrive(&bars->s_free[sb]);
        float x[128];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          x[i] = i < nv ? __uint_as_float(r[i]) * a.sl2 : -INFINITY;
          mx = fmaxf(mx, x[i]);
        }
        const float m_new = fmaxf(m, mx);
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
          // O holds blocks < j: wait for the last PV, then rescale it in TMEM.
          const uint32_t pi = it - 1;
          if (!(ok = warp_wait(&bars->pv_done[pi & 1], (pi >> 1) & 1, abort))) break;
          tc_fence_after();
          const float alpha = ex2(m - m_new);
          uint32_t o[128];
          tmem_ld128(tmem + lane_addr + kColO, o);
#pragma unroll
          for (int i = 0; i < 128; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_st32(tmem + lane_addr + kColO + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&o[c * 32]));
          tmem_st_wait();
          l *= alpha;
          m = m_new;
        }
        // P_j into TMEM buffer pb once the PV that last read that buffer is done.
        const uint32_t pb = it & 1, pu = it >> 1;
        if (!(ok = warp_wait(&bars->pv_done[pb], (pu & 1) ^ 1, abort))) break;
        tc_fence_after();
        uint32_t pk[64];
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float p0 = ex2(x[2 * i] - m), p1 = ex2(x[2 * i + 1] - m);
          sum += p0 + p1;
          pk[i] = pack_bf16(p0, p1);
        }
        l += sum;
        tmem_st32(tmem + lane_addr + kColP + pb * 64, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(tmem + lane_addr + kColP + pb * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
        tmem_st_wait();
        if (nv < 128) {
          // V rows past the valid keys may hold anything (P is 0 there, but
          // 0 * NaN is not 0): zero them before the PV MMA reads the stage.
          const uint32_t s = it % kKVStages, u = it / kKVStages;
          if (!(ok = warp_wait(&bars->v_full[s], u & 1, abort))) break;
          if (row >= nv) {
            uint4* v0 = reinterpret_cast<uint4*>(sm + kOffV + s * kTileBytes + row * 128);
            uint4* v1 = reinterpret_cast<uint4*>(sm + kOffV + s * kTileBytes + kRegionBytes + row * 128);
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              v0[c] = z;
              v1[c] = z;
            }
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&bars->p_full[pb]);
      }
      if (!ok) break;
      // Epilogue: O / l -> bf16 -> out.
      const uint32_t last = it - 1;
      if (!(ok = warp_wait(&bars->pv_done[last & 1], (last >> 1) & 1, abort))) break;
      tc_fence_after();
      uint32_t o[128];
      tmem_ld128(tmem + lane_addr + kColO, o);
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      const float inv = 1.f / l;
      const int64_t q = int64_t(t.qt) * 128 + row;
      if (q < a.Lq) {
        uint4* dst = reinterpret_cast<uint4*>(a.out + (int64_t(t.lh) * a.Lq + q) * 128);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
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
  if (warp == 5) {
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
