// Step 5 over the e4m3 compressed cache, on the tensor cores with
// kind::f8f6f4 (Forcing-KV, ai-feeds.com/i/paper/2605.09681:
// "输出与工程收益" -- the compressed KV replaces the cache inside attention;
// "与现有产品/工作流的接口" item 3 -- it composes with KV quantization).
//
// out_i = sum_j softmax_j(scale * q~_i . k~_j) v~_j, where x~ = e4m3(code) *
// scale of its block: one scale per query row (sq), per key segment (sk) and
// per value segment (sv), a segment being a kept history frame or a chunk
// frame.  Keys = kept rows of the compressed cache then the chunk's rows, no
// causal mask; fp32 accumulation; bf16 out.
//
// The unit, stream and warp-role structure is that of the bf16 kernel (two
// interleaved key-block streams per 128-query tile, softmax warpgroups 0-1,
// TMA warp 8, MMA warp 9, P aliasing S in TMEM); what differs:
//   * operand tiles are [128][128] bytes, one 128-byte swizzle atom per row,
//     one TMA box each; Q and K are K-major, V row-major (MN-major B of the
//     P.V product); an MMA step covers K = 32;
//   * the scales never touch the tensor core.  A 128-key block spans at most
//     two segments (T >= 128), and for each segment g the softmax uses
//       x_j = S_j * (sq_i * sk_g * scale * log2 e) + log2(sv_g / sv_max)
//     so one FMA per logit (as in the bf16 kernel) both dequantises the
//     logit and folds the value scale into the probability P'_j = 2^(x_j - m);
//     sv_max = the largest value scale of the head keeps P' <= 2^8 (lazy
//     rescale bound).  P' is rounded to e4m3 into TMEM; the row sum is
//     l = sum_g (sv_max / sv_g) sum_{j in g} P'_j, the sum of the unscaled
//     probabilities; the output is sv_max * (P'.v) / l;
//   * 4 shared-memory stages of K and of V (the tiles are half as large).
#include <cuda_fp8.h>

#include "fkv_internal.cuh"
#include "sm100_common.cuh"
#include "f8_common.cuh"
#include "attend_common.cuh"

namespace fkv {
namespace sm100 {
namespace f8 {

constexpr uint32_t kTile = 128 * 128;  // bytes of one e4m3 [128][128] tile
constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(kThreads * kLaunchRegs >= 256 * kSoftmaxRegs + 128 * kControlRegs,
              "register split exceeds the launch allocation");
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr float kRescaleLog2 = 8.0f;
// One of every FKV_F8_POLY_EVERY exponential pairs of a block goes to the
// FMA-pipe exp2_poly2 instead of the MUFU unit (0: none; 4 measured best at
// 480P: 0.603 ms against 0.619 with none, 0.614 with 3, 0.644 with 2).
#ifndef FKV_F8_POLY_EVERY
#define FKV_F8_POLY_EVERY 4
#endif
constexpr int kPolyEvery = FKV_F8_POLY_EVERY;

constexpr uint32_t kIdescQK = idesc_e4m3(128, 128, false);
constexpr uint32_t kIdescPV = idesc_e4m3(128, 128, true);

__host__ __device__ constexpr uint32_t col_s(int h) { return 128u * uint32_t(h); }
__host__ __device__ constexpr uint32_t col_o(int h) { return 256u + 128u * uint32_t(h); }

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kOffBar = kOffV + kStages * kTile;

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kStages], k_empty[kStages];
  uint64_t v_full[kStages], v_empty[kStages];
  uint64_t s_full[2], p_full[2];
  uint64_t o_ready, o_free;
  uint64_t mma_done;
  uint64_t x_full, x_read;
  uint32_t tmem_base;
  int abort;
  float2 xml[2][128];
};
constexpr size_t kSmem = kOffBar + sizeof(Bars) + 1024;  // + slack to align the base
static_assert(kSmem <= 232448, "shared memory above the per-CTA limit");

struct Args {
  int64_t Lq, comp_rows, seg_len, max_kept;
  int n_qtiles, n_tiles, Fc;
  float sl2;  // scale * log2(e)
  const int32_t* kept_cnt;
  const float* sk_comp;  // [LH][max_kept]
  const float* sv_comp;
  const float* sk_cur;   // [LH][Fc]
  const float* sv_cur;
  const float* sq;       // [LH][Lq]
  __nv_bfloat16* out;
  int32_t* status;
};

#ifndef FKV_F8_ISSUE_LOOKAHEAD
#define FKV_F8_ISSUE_LOOKAHEAD 0
#endif

// Four probabilities -> four e4m3 codes in one 32-bit word, the first in the low byte.
__device__ __forceinline__ uint32_t pack_e4m3x4(float2 a, float2 b) {
  const uint32_t lo = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
  const uint32_t hi = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
  return lo | (hi << 16);
}

__global__ void __launch_bounds__(kThreads, 1)
attend_fp8_kernel(const __grid_constant__ CUtensorMap tm_q,
                  const __grid_constant__ CUtensorMap tm_kc,
                  const __grid_constant__ CUtensorMap tm_vc,
                  const __grid_constant__ CUtensorMap tm_kn,
                  const __grid_constant__ CUtensorMap tm_vn, const Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  Bars* bars = reinterpret_cast<Bars*>(sm + kOffBar);
  volatile int* abort = &bars->abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bars->s_full[h], 1);
      mbar_init(&bars->p_full[h], 128);
    }
    mbar_init(&bars->o_ready, 1);
    mbar_init(&bars->o_free, kSoftmaxThreads);
    mbar_init(&bars->mma_done, 1);
    mbar_init(&bars->x_full, kSoftmaxThreads);
    mbar_init(&bars->x_read, kSoftmaxThreads);
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
  // Everything above is on-chip; global memory is touched only once the
  // kernel before this one has completed (programmatic dependent launch).
  pdl_wait();
  if (warp >= 8) {
    regs_decrease<kControlRegs>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0 || lane == 1) {  // lane 0: Q and K; lane 1: V
      const bool is_k = lane == 0;
      if (is_k) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_kc);
        prefetch_tmap(&tm_kn);
      } else {
        prefetch_tmap(&tm_vc);
        prefetch_tmap(&tm_vn);
      }
      uint64_t* full = is_k ? bars->k_full : bars->v_full;
      uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
      const CUtensorMap* mA = is_k ? &tm_kc : &tm_vc;
      const CUtensorMap* mB = is_k ? &tm_kn : &tm_vn;
      uint8_t* ring = sm + (is_k ? kOffK : kOffV);
      uint32_t n = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const Unit t = decode(a, tile);
        if (is_k) {
          if (!(ok = mbar_wait(&bars->q_empty, (tc & 1) ^ 1, abort))) break;
          mbar_expect_tx(&bars->q_full, kTile);
          tma_load_3d(sm + kOffQ, &tm_q, &bars->q_full, 0, t.qt * 128, t.lh);
          ++tc;
        }
        for (int j = 0; ok && j < t.nb0; ++j) {
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && j >= t.nb1) break;
            const int b = block_of(t, h, j);
            const bool inA = b < t.nbA;
            const int row = (inA ? b : b - t.nbA) * 128;
            const uint32_t s = n % kStages, u = n / kStages;
            if (!(ok = mbar_wait(&empty[s], (u & 1) ^ 1, abort))) break;
            mbar_expect_tx(&full[s], kTile);
            tma_load_3d(ring + s * kTile, inA ? mA : mB, &full[s], 0, row, t.lh);
            ++n;
          }
        }
      }
      for (uint32_t i = n > kStages ? n - kStages : 0; i < n; ++i)
        drain_wait(&full[i % kStages], (i / kStages) & 1);
      if (is_k && tc > 0) drain_wait(&bars->q_full, (tc - 1) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // One thread issues the MMAs only slightly faster than the tensor core
    // runs them and the hardware queue is short, so this thread only waits
    // and issues: ring cursors (K and V are consumed in load order),
    // precomputed descriptors, one commit per S group (the softmax releases
    // the K and V stages), a tcgen05 fence only after P and O handoffs.
    if (lane == 0) {
      uint32_t uc = 0, ks = 0, kph = 0, vs = 0, vph = 0;
      uint32_t p_use[2] = {0, 0};
      bool ok = true;
      bool kf_ok = false, vf_ok = false;  // next K / V stage seen complete ahead of use
      const uint64_t dq = kmajor8_desc(smem_u32(sm + kOffQ), 0);
      const uint64_t dk0 = kmajor8_desc(smem_u32(sm + kOffK), 0);
      const uint64_t dv0 = mnmajor8_desc(smem_u32(sm + kOffV), 0);
      constexpr uint32_t kStageDesc = kTile >> 4;  // descriptor step between ring stages
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++uc) {
        const Unit t = decode(a, tile);
        bool o_free_seen = false;
        // O_h += P_h V for the stream's next block (`first`: its first of the unit).
        auto issue_pv = [&](int h, bool first) -> bool {
          if (!o_free_seen) {
            if (!mbar_wait(&bars->o_free, (uc & 1) ^ 1, abort)) return false;
            o_free_seen = true;
          }
          if (!vf_ok && !mbar_wait(&bars->v_full[vs], vph, abort)) return false;
          if (!mbar_wait(&bars->p_full[h], p_use[h] & 1, abort)) return false;
          ++p_use[h];
          tc_fence_after();
          // step k: 32 keys = 4 KB further (descriptor address field: bytes >> 4)
          const uint64_t dv = dv0 + uint64_t(vs * kStageDesc);
#if FKV_F8_ISSUE_LOOKAHEAD
          // K and V stages are consumed in load order: test the K stage of the
          // S group that comes next while these MMAs issue
          kf_ok = mma4_ts_e4m3_probe(tmem + col_o(h), tmem + col_s(h), dv, kIdescPV,
                                     first ? 0u : 1u, &bars->k_full[ks], kph) != 0;
#else
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts_e4m3(tmem + col_o(h), tmem + col_s(h) + k * 8, dv + uint64_t(k) * 256u,
                        kIdescPV, (first && k == 0) ? 0u : 1u);
#endif
          vf_ok = false;
          if (++vs == kStages) { vs = 0; vph ^= 1; }
          return true;
        };
        // S_h = Q K^T for the stream's next block; step k: 32 bytes along the row.
        auto issue_s = [&](int h) -> bool {
          if (!kf_ok && !mbar_wait(&bars->k_full[ks], kph, abort)) return false;
          kf_ok = false;
          const uint64_t dk = dk0 + uint64_t(ks * kStageDesc);
#if FKV_F8_ISSUE_LOOKAHEAD
          // ... and the V stage of the P.V group that comes next
          vf_ok = mma4_ss_e4m3_probe(tmem + col_s(h), dq, dk, kIdescQK, 0u, &bars->v_full[vs],
                                     vph) != 0;
#else
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ss_e4m3(tmem + col_s(h), dq + uint64_t(2 * k), dk + uint64_t(2 * k), kIdescQK,
                        k > 0 ? 1u : 0u);
#endif
          mma_commit(&bars->s_full[h]);
          if (++ks == kStages) { ks = 0; kph ^= 1; }
          return true;
        };
        if (!(ok = mbar_wait(&bars->q_full, uc & 1, abort))) break;
        // Per step j: PV_0(j-1), S_0(j), PV_1(j-1), S_1(j) -- the load order of K
        // and of V; where stream 1 has one block fewer, its last PV follows S_0
        // of the extra block, again in load order.
        for (int j = 0; ok && j < t.nb0; ++j) {
          if (j > 0 && !(ok = issue_pv(0, j == 1))) break;
          if (!(ok = issue_s(0))) break;
          if (j < t.nb1) {
            if (j > 0 && !(ok = issue_pv(1, j == 1))) break;
            if (!(ok = issue_s(1))) break;
          } else if (j == t.nb1 && j > 0) {
            if (!(ok = issue_pv(1, j == 1))) break;
          }
        }
        if (!ok) break;
        mma_commit(&bars->q_empty);
        if (!(ok = issue_pv(0, t.nb0 == 1))) break;
        if (t.nb1 == t.nb0 && t.nb1 > 0 && !(ok = issue_pv(1, t.nb1 == 1))) break;
        mma_commit(&bars->o_ready);
      }
      mma_commit(&bars->mma_done);
      drain_wait(&bars->mma_done, 0);
    }
  }
  } else {
    regs_increase<kSoftmaxRegs>();
    // ------------------------------------------------------------ softmax warpgroups
    const int h = warp >> 2;                    // stream
    const int row = threadIdx.x & 127;          // query row = TMEM lane
    const uint32_t lane_addr = uint32_t((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_addr + col_s(h);
    const int64_t T = a.seg_len;
    uint32_t use = 0, base = 0, uc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++uc) {
      const Unit t = decode(a, tile);
      const int mine = h ? t.nb1 : t.nb0;
      const int64_t q = int64_t(t.qt) * 128 + row;
      // rows past Lq (zero-filled by the copy) are computed but never written
      const float cq = (q < a.Lq ? __ldg(a.sq + int64_t(t.lh) * a.Lq + q) : 1.f) * a.sl2;
      const float* skA = a.sk_comp + int64_t(t.lh) * a.max_kept;
      const float* svA = a.sv_comp + int64_t(t.lh) * a.max_kept;
      const float* skB = a.sk_cur + int64_t(t.lh) * a.Fc;
      const float* svB = a.sv_cur + int64_t(t.lh) * a.Fc;
      // sv_max over the segments this unit reads (scales are > 0)
      const int nsegA = int((t.nA + T - 1) / T);
      float svm = 0.f;
      for (int g = lane; g < nsegA; g += 32) svm = fmaxf(svm, __ldg(svA + g));
      for (int g = lane; g < a.Fc; g += 32) svm = fmaxf(svm, __ldg(svB + g));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) svm = fmaxf(svm, __shfl_xor_sync(0xffffffffu, svm, o));
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < mine; ++j, ++use) {
        const int b = block_of(t, h, j);
        const bool inA = b < t.nbA;
        const int64_t row0 = int64_t(inA ? b : b - t.nbA) * 128;
        const int64_t rows_left = (inA ? t.nA : a.Lq) - row0;
        const int nv = rows_left < 128 ? int(rows_left) : 128;  // valid keys of the block
        const int g0 = int(row0 / T);
        const int bc = int((g0 + 1) * T - row0);  // first column of segment g0 + 1
        const bool split = bc < nv;               // warp-uniform
        const float* sk = inA ? skA : skB;
        const float* sv = inA ? svA : svB;
        const float sk0 = __ldg(sk + g0), sv0 = __ldg(sv + g0);
        const float sk1 = split ? __ldg(sk + g0 + 1) : sk0;
        const float sv1 = split ? __ldg(sv + g0 + 1) : sv0;
        const float ck0 = cq * sk0, ck1 = cq * sk1;
        const float corr0 = svm / sv0, corr1 = svm / sv1;   // >= 1
        const float lsv0 = -__log2f(corr0), lsv1 = -__log2f(corr1);
        if (!(ok = warp_wait(&bars->s_full[h], use & 1, abort))) break;
        if (row == 0) {
          // S_h(j) is complete, and with it every MMA issued before it: the K
          // stage it read and the V stage of this stream's previous PV are free.
          mbar_arrive(&bars->k_empty[(base + uint32_t(seq_pos(t, h, j))) % kStages]);
          if (j > 0) mbar_arrive(&bars->v_empty[(base + uint32_t(seq_pos(t, h, j - 1))) % kStages]);
        }
        tc_fence_after();
        uint32_t sr[128];  // raw fp32 logits of this row (e4m3 codes' dot products)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_ld_wait();
        if (nv < 128) {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= nv) sr[i] = 0xff800000u;  // -inf
        }
#define SV(i) __uint_as_float(sr[i])
        if (split) {  // per-column constants: x = S * ck + lsv in place
#pragma unroll
          for (int i = 0; i < 128; ++i)
            sr[i] = __float_as_uint(i < bc ? fmaf(SV(i), ck0, lsv0) : fmaf(SV(i), ck1, lsv1));
        }
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(SV(k), SV(k + 8));
#pragma unroll
        for (int i = 16; i < 128; i += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], SV(i + k), SV(i + k + 8));
        const float bmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]),
                                 fmaxf(mx[6], mx[7]));
        const float m_new = fmaxf(m, split ? bmax : fmaf(bmax, ck0, lsv0));  // ck0 > 0
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
          const float alpha = ex2(m - m_new);
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t o[16];
            tmem_ld16(tmem + lane_addr + col_o(h) + c * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(tmem + lane_addr + col_o(h) + c * 16, o);
          }
          tmem_st_wait();
          l *= alpha;
          m = m_new;
        }
        uint32_t pk[32];  // P' as e4m3, 4 keys per 32-bit TMEM column
        if (!split) {
          float2 acc[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
          const float2 ck2 = make_float2(ck0, ck0), off2 = make_float2(lsv0 - m, lsv0 - m);
#pragma unroll
          for (int w = 0; w < 32; ++w) {
            const float2 e0 = ffma2(make_float2(SV(4 * w), SV(4 * w + 1)), ck2, off2);
            const float2 e1 = ffma2(make_float2(SV(4 * w + 2), SV(4 * w + 3)), ck2, off2);
            const bool poly0 = kPolyEvery > 0 && (2 * w) % (kPolyEvery > 0 ? kPolyEvery : 1) ==
                                                     (kPolyEvery > 0 ? kPolyEvery : 1) - 1;
            const bool poly1 = kPolyEvery > 0 && (2 * w + 1) % (kPolyEvery > 0 ? kPolyEvery : 1) ==
                                                     (kPolyEvery > 0 ? kPolyEvery : 1) - 1;
            const float2 p0 = poly0 ? exp2_poly2(e0) : make_float2(ex2(e0.x), ex2(e0.y));
            const float2 p1 = poly1 ? exp2_poly2(e1) : make_float2(ex2(e1.x), ex2(e1.y));
            acc[w & 3] = fadd2(acc[w & 3], fadd2(p0, p1));
            pk[w] = pack_e4m3x4(p0, p1);
          }
          const float2 s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
          l = fmaf(s2.x + s2.y, corr0, l);
        } else {
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int w = 0; w < 32; ++w) {
            float p[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              p[k] = ex2(SV(4 * w + k) - m);
              if (4 * w + k < bc) s0 += p[k]; else s1 += p[k];
            }
            pk[w] = pack_e4m3x4(make_float2(p[0], p[1]), make_float2(p[2], p[3]));
          }
          l = fmaf(s0, corr0, fmaf(s1, corr1, l));
        }
#undef SV
        tmem_st32(tS, pk);
        tmem_st_wait();
        if (nv < 128) {
          // V rows past the valid keys may hold anything (P' is 0 there, but
          // 0 * NaN is not 0): zero them before the PV MMA reads the stage.
          const uint32_t pos = base + uint32_t(seq_pos(t, h, j));
          const uint32_t s = pos % kStages, u = pos / kStages;
          if (!(ok = warp_wait(&bars->v_full[s], u & 1, abort))) break;
          if (row >= nv) {
            uint4* v0 = reinterpret_cast<uint4*>(sm + kOffV + s * kTile + row * 128);
            const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int c = 0; c < 8; ++c) v0[c] = z;
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&bars->p_full[h]);
      }
      if (!ok) break;
      // V stage of this stream's last PV (released once both PV chains are done)
      const uint32_t last_v = mine > 0 ? (base + uint32_t(seq_pos(t, h, mine - 1))) % kStages : 0u;
      base += uint32_t(t.nb);
      // ---- merge the two streams and write this thread's 64 output columns
      if (!(ok = warp_wait(&bars->o_ready, uc & 1, abort))) break;
      if (row == 0 && mine > 0) mbar_arrive(&bars->v_empty[last_v]);
      tc_fence_after();
      if (!(ok = warp_wait(&bars->x_read, (uc & 1) ^ 1, abort))) break;  // last unit's reads done
      bars->xml[h][row] = make_float2(m, l);
      mbar_arrive(&bars->x_full);
      if (!(ok = warp_wait(&bars->x_full, uc & 1, abort))) break;
      const float2 other = bars->xml[h ^ 1][row];
      mbar_arrive(&bars->x_read);
      const float m0 = h ? other.x : m, l0 = h ? other.y : l;
      const float m1 = h ? m : other.x, l1 = h ? l : other.y;
      const bool two = t.nb1 > 0;
      const float M = two ? fmaxf(m0, m1) : m0;
      const float a0 = ex2(m0 - M), a1 = two ? ex2(m1 - M) : 0.f;
      const float inv = svm / (l0 * a0 + (two ? l1 * a1 : 0.f));
      const float c0 = a0 * inv, c1 = a1 * inv;
      uint4* dst = reinterpret_cast<uint4*>(a.out + (int64_t(t.lh) * a.Lq + q) * 128 + h * 64);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r0[32], r1[32];
        tmem_ld32(tmem + lane_addr + col_o(0) + h * 64 + c * 32, r0);
        if (two) tmem_ld32(tmem + lane_addr + col_o(1) + h * 64 + c * 32, r1);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0 = __uint_as_float(r0[2 * i]) * c0, x1 = __uint_as_float(r0[2 * i + 1]) * c0;
          if (two) {
            x0 = fmaf(__uint_as_float(r1[2 * i]), c1, x0);
            x1 = fmaf(__uint_as_float(r1[2 * i + 1]), c1, x1);
          }
          w[i] = pack_bf16(x0, x1);
        }
        if (q < a.Lq) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[c * 4 + k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->o_free);
    }
  }

  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && bars->abort) report(a.status, FKV_ERR_TIMEOUT, blockIdx.x);
}

}  // namespace f8
}  // namespace sm100

cudaError_t launch_attend_fp8_sm100(const Dims& d, const fkv_fp8_cache_t& c,
                                    const int32_t* kept_cnt, void* out, int32_t* status,
                                    cudaStream_t s) {
  using namespace sm100;
  using namespace sm100::f8;
  const uint64_t row_b = 128;
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  if (!make_tmap_u8(&tq, c.q_cur, d.Lq, d.LH, row_b, d.Lq * row_b) ||
      !make_tmap_u8(&tkn, c.k_cur, d.Lq, d.LH, row_b, d.Lq * row_b) ||
      !make_tmap_u8(&tvn, c.v_cur, d.Lq, d.LH, row_b, d.Lq * row_b))
    return cudaErrorInvalidValue;
  if (d.comp_rows > 0) {
    if (!make_tmap_u8(&tkc, c.k_comp, d.comp_rows, d.LH, row_b, d.comp_rows * row_b) ||
        !make_tmap_u8(&tvc, c.v_comp, d.comp_rows, d.LH, row_b, d.comp_rows * row_b))
      return cudaErrorInvalidValue;
  } else {  // no compressed rows: never read, any valid map will do
    tkc = tkn;
    tvc = tvn;
  }
  Args a;
  a.Lq = d.Lq;
  a.comp_rows = d.comp_rows;
  a.seg_len = d.seg_len;
  a.max_kept = d.max_kept;
  a.n_qtiles = int((d.Lq + 127) / 128);
  a.n_tiles = a.n_qtiles * d.LH;
  a.Fc = d.Fc;
  a.sl2 = d.scale * 1.4426950408889634f;
  a.kept_cnt = kept_cnt;
  a.sk_comp = c.k_comp_scale;
  a.sv_comp = c.v_comp_scale;
  a.sk_cur = c.k_cur_scale;
  a.sv_cur = c.v_cur_scale;
  a.sq = c.q_scale;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.status = status;
  cudaError_t e = cudaFuncSetAttribute(attend_fp8_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
  if (e != cudaSuccess) return e;
  const int grid = a.n_tiles < num_sms() ? a.n_tiles : num_sms();
  return launch_kernel(attend_fp8_kernel, dim3(grid), dim3(kThreads), kSmem, s, d.pdl, tq, tkc,
                       tvc, tkn, tvn, a);
}

}  // namespace fkv
