// Step 5 on the tensor cores: the chunk's queries attend to the compressed
// history followed by the chunk's own keys (Forcing-KV,
// ai-feeds.com/i/paper/2605.09681, "输出与工程收益": the compressed KV
// replaces the cache inside attention; "与现有产品/工作流的接口" step 2).
//
// out_i = sum_j softmax_j(scale * q_i . k_j) v_j over keys = k_comp rows
// [0, kept rows) then k_cur rows [0, Lq), no causal mask; bf16 in, fp32
// accumulation, bf16 out.
//
// Work unit = one 128-query tile of one (layer, head); one persistent CTA per
// SM walks the units.  Inside a unit the 128-key blocks are split between two
// streams h = 0, 1 (first and second half of the blocks) that run
// interleaved on the tensor core, each with its own softmax warpgroup, logit
// tile S_h and fp32 accumulator O_h in TMEM; at the end of the unit the two
// partial softmaxes are merged (rescaled by their row maxima).  While one
// warpgroup computes exponentials the tensor core works on the other
// stream's MMAs.
//
// Warp roles (384 threads; warps 10-11 only complete the control warpgroup):
//   warps 0-3 / 4-7  softmax of stream 0 / 1: thread t owns query row t
//              (= TMEM lane t).  Reads S_h from TMEM, keeps the running row
//              max m (base-2 logits) and sum l, writes P = 2^(S*scale*log2e
//              - m) as bf16 pairs into the first 64 columns of S_h, and
//              rescales O_h in TMEM only when m grows by more than 2^8 (lazy
//              rescaling: P stays <= 256, exact after the final merge).
//              Exponentials run on the MUFU unit, except one pair in
//              FKV_POLY_EVERY (8) that goes to the FMA-pipe polynomial
//              exp2_poly2 (fastest of 3 ... 16 at 480P).  The lead thread of
//              each warpgroup releases the K stage of S_h(j) and the V stage
//              of PV_h(j-1) once it sees S_h(j) complete.
//   warp 8     TMA: lane 0 loads Q (once per unit) and the K blocks, lane 1
//              the V blocks, into rings (3 + 3 stages) in the order the MMAs
//              use them: stream 0 block j, stream 1 block j, stream 0 block
//              j+1...
//   warp 9     MMA issuer (one thread) and TMEM owner.  Per step j it issues
//              O_0 += P_0 V (block j-1), S_0 = Q K^T (block j), then the same
//              for stream 1.  tcgen05 MMAs of one thread execute in issue
//              order, so S_h of block j overwrites P_h only after the PV that
//              reads it, and by the time S_h is complete the previous PV into
//              O_h is complete too (the softmax may rescale O_h right away).
//              The issuing thread issues an M=128, N=128, K=16 MMA only
//              slightly faster than the tensor core executes one and the
//              hardware queue is short, so its work between MMA groups (each
//              mbarrier test or commit costs it ~90 cycles) idles the tensor
//              core; it is kept to one wait and one commit per group.
// TMEM (512 columns): S_0 [0,128), S_1 [128,256), O_0 [256,384), O_1 [384,512).
//
// Key blocks past the valid rows of a range are masked (logit -> -inf) and
// their V rows zeroed in shared memory before use, so compressed-cache rows
// past the kept count are never read as data, whatever they hold.  Every
// mbarrier wait is bounded; on timeout the CTA records FKV_ERR_TIMEOUT, waits
// (bounded) for its own copies and MMAs, frees TMEM and returns.
#include "fkv_internal.cuh"
#include "sm100_common.cuh"
#include "attend_common.cuh"

namespace fkv {
namespace sm100 {

// The MMA issuer tests the next group's K / V barrier inside the current
// group's MMA issue (1) or waits on it in front of the next group (0).
#ifndef FKV_ISSUE_LOOKAHEAD
#define FKV_ISSUE_LOOKAHEAD 1
#endif
#ifndef FKV_ATTN_K_STAGES
#define FKV_ATTN_K_STAGES 3
#endif
#ifndef FKV_ATTN_V_STAGES
#define FKV_ATTN_V_STAGES 3
#endif
// Ring depths of the K and V tiles (K + V = 6 tiles of 32 KB fit beside Q).
constexpr int kKStages = FKV_ATTN_K_STAGES;
constexpr int kVStages = FKV_ATTN_V_STAGES;
constexpr int kAttnThreads = 384;        // 3 warpgroups
// Register split (setmaxnreg): the kernel is launched with kLaunchRegs per
// thread; the control warpgroup (TMA, MMA, two idle warps) gives registers
// back, the two softmax warpgroups take them.  Budget check, registers per
// CTA: 384 * 168 = 64512 at launch >= 256 * 224 + 128 * 56 = 64512 after;
// per SM sub-partition (one warp of each warpgroup): (224+224+56) * 32 =
// 16128 <= 16384.
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kControlRegs = 56;
static_assert(kAttnThreads * kLaunchRegs >= 256 * kSoftmaxRegs + 128 * kControlRegs,
              "register split exceeds the launch allocation");
constexpr int kSoftmaxThreads = 256;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kIdescQK = idesc_bf16(128, 128, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 128, true);
constexpr float kRescaleLog2 = 8.0f;
static_assert(kProductionWaitCycles == kWaitCycles, "one production wait limit");
// One of every FKV_POLY_EVERY exponential pairs goes to the FMA-pipe exp2 (0: none).
#ifndef FKV_POLY_EVERY
#define FKV_POLY_EVERY 8
#endif

__host__ __device__ constexpr uint32_t col_s(int h) { return 128u * uint32_t(h); }
__host__ __device__ constexpr uint32_t col_o(int h) { return 256u + 128u * uint32_t(h); }

constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kTileBytes;
constexpr uint32_t kOffV = kOffK + kKStages * kTileBytes;
constexpr uint32_t kOffBar = kOffV + kVStages * kTileBytes;

struct AttnBars {
  uint64_t q_full, q_empty;
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t s_full[2], p_full[2];  // per stream
  uint64_t o_ready, o_free;       // per unit: both PV chains done / both O read
  uint64_t mma_done;
  uint64_t x_full, x_read;        // merge exchange handshake (256 arrivals each)
  uint32_t tmem_base;
  int abort;
  float2 xml[2][128];             // [stream][row] (row max, row sum) for the merge
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
  long long wait_cycles;  // limit of every bounded wait (kWaitCycles in production)
  int withhold_s0;        // diagnostic: CTA 0 withholds the completion signal of its
                          // first S_0 group (0 in production)
};

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
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
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
  // Everything above is on-chip; global memory (kept counts, Q/K/V, the
  // output) is touched only once the kernel before this one has completed.
  pdl_wait();
  if (warp >= 8) {
    regs_decrease<kControlRegs>();
  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    if (lane == 0) {  // Q and K
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_kc);
      prefetch_tmap(&tm_kn);
      uint32_t n = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const Unit t = decode(a, tile);
        if (!(ok = mbar_wait(&bars->q_empty, (tc & 1) ^ 1, abort, a.wait_cycles))) break;
        mbar_expect_tx(&bars->q_full, kTileBytes);
        tma_load_tile(sm + kOffQ, &tm_q, &bars->q_full, t.qt * 128, t.lh);
        ++tc;
        for (int j = 0; ok && j < t.nb0; ++j) {
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && j >= t.nb1) break;
            const int b = block_of(t, h, j);
            const bool inA = b < t.nbA;
            const int row = (inA ? b : b - t.nbA) * 128;
            const uint32_t s = n % kKStages, u = n / kKStages;
            if (!(ok = mbar_wait(&bars->k_empty[s], (u & 1) ^ 1, abort, a.wait_cycles))) break;
            mbar_expect_tx(&bars->k_full[s], kTileBytes);
            tma_load_tile(sm + kOffK + s * kTileBytes, inA ? &tm_kc : &tm_kn, &bars->k_full[s],
                          row, t.lh);
            ++n;
          }
        }
      }
      for (uint32_t i = n > kKStages ? n - kKStages : 0; i < n; ++i)
        drain_wait(&bars->k_full[i % kKStages], (i / kKStages) & 1);
      if (tc > 0) drain_wait(&bars->q_full, (tc - 1) & 1);
    } else if (lane == 1) {  // V
      prefetch_tmap(&tm_vc);
      prefetch_tmap(&tm_vn);
      uint32_t n = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x) {
        const Unit t = decode(a, tile);
        for (int j = 0; ok && j < t.nb0; ++j) {
          for (int h = 0; h < 2; ++h) {
            if (h == 1 && j >= t.nb1) break;
            const int b = block_of(t, h, j);
            const bool inA = b < t.nbA;
            const int row = (inA ? b : b - t.nbA) * 128;
            const uint32_t s = n % kVStages, u = n / kVStages;
            if (!(ok = mbar_wait(&bars->v_empty[s], (u & 1) ^ 1, abort, a.wait_cycles))) break;
            mbar_expect_tx(&bars->v_full[s], kTileBytes);
            tma_load_tile(sm + kOffV + s * kTileBytes, inA ? &tm_vc : &tm_vn, &bars->v_full[s],
                          row, t.lh);
            ++n;
          }
        }
      }
      for (uint32_t i = n > kVStages ? n - kVStages : 0; i < n; ++i)
        drain_wait(&bars->v_full[i % kVStages], (i / kVStages) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // The tensor core queues only a few MMAs and one thread issues them barely
    // faster than they execute, so whatever this thread does between two MMA
    // groups leaves the tensor core idle.  It therefore only waits and
    // issues: ring stages advance by cursors (K and V are consumed in load
    // order), descriptors are precomputed, one commit per S group (the
    // softmax releases the K and V stages), and a tcgen05 fence only where
    // another thread wrote TMEM (P, and O after the epilogue).
    if (lane == 0) {
      uint32_t uc = 0, ks = 0, kph = 0, vs = 0, vph = 0;
      uint32_t p_use[2] = {0, 0};
      bool ok = true;
      // Diagnostic only: one software arrival that never comes, so that the
      // softmax's bounded wait on it runs out (the MMAs themselves are issued
      // and complete; nothing else is left outstanding behind the signal).
      bool withhold = a.withhold_s0 != 0 && blockIdx.x == 0;
      bool kf_ok = false, vf_ok = false;  // next K / V stage seen complete ahead of use
      const uint64_t dq = kmajor_desc(smem_u32(sm + kOffQ), 0);
      const uint64_t dk0 = kmajor_desc(smem_u32(sm + kOffK), 0);
      const uint64_t dv0 = mnmajor_desc(smem_u32(sm + kOffV), 0);
      constexpr uint32_t kStageDesc = kTileBytes >> 4;  // descriptor step between ring stages
      for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++uc) {
        const Unit t = decode(a, tile);
        bool o_free_seen = false;
        // O_h += P_h V for the stream's next block (`first`: its first of the unit).
        // K and V stages are consumed in load order, so the K stage of the S
        // group that follows a PV group, and the V stage of the PV group that
        // follows an S group, are known in advance: each group tests that
        // stage's barrier without blocking, inside its own MMA issue (kf_ok /
        // vf_ok), and the next group waits only when the test saw it pending.
#if FKV_ISSUE_LOOKAHEAD
        auto issue_pv = [&](int h, bool first) -> bool {
          if (!o_free_seen) {
            if (!mbar_wait(&bars->o_free, (uc & 1) ^ 1, abort, a.wait_cycles)) return false;
            o_free_seen = true;
          }
          if (!vf_ok && !mbar_wait(&bars->v_full[vs], vph, abort, a.wait_cycles)) return false;
          if (!mbar_wait(&bars->p_full[h], p_use[h] & 1, abort, a.wait_cycles)) return false;
          ++p_use[h];
          tc_fence_after();
          // step k: P columns 8k.., V rows 16k.. (2048 B = 128 descriptor units)
          kf_ok = mma8_ts_probe(tmem + col_o(h), tmem + col_s(h),
                                dv0 + uint64_t(vs * kStageDesc), kIdescPV, first ? 0u : 1u,
                                &bars->k_full[ks], kph) != 0;
          vf_ok = false;
          if (++vs == kVStages) { vs = 0; vph ^= 1; }
          return true;
        };
        // S_h = Q K^T for the stream's next block.
        auto issue_s = [&](int h) -> bool {
          if (!kf_ok && !mbar_wait(&bars->k_full[ks], kph, abort, a.wait_cycles)) return false;
          kf_ok = false;
          // step k of the 128-deep contraction: 32 bytes along a 128-byte
          // swizzled row, then the second 64-column region
          vf_ok = mma8_ss_probe(tmem + col_s(h), dq, dk0 + uint64_t(ks * kStageDesc), kIdescQK,
                                0u, &bars->v_full[vs], vph) != 0;
          if (withhold && h == 0) withhold = false;
          else mma_commit(&bars->s_full[h]);
          if (++ks == kKStages) { ks = 0; kph ^= 1; }
          return true;
        };
#else
        auto issue_pv = [&](int h, bool first) -> bool {
          if (!o_free_seen) {
            if (!mbar_wait(&bars->o_free, (uc & 1) ^ 1, abort, a.wait_cycles)) return false;
            o_free_seen = true;
          }
          if (!mbar_wait(&bars->v_full[vs], vph, abort, a.wait_cycles)) return false;
          if (!mbar_wait(&bars->p_full[h], p_use[h] & 1, abort, a.wait_cycles)) return false;
          ++p_use[h];
          tc_fence_after();
          const uint64_t dv = dv0 + uint64_t(vs * kStageDesc);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ts(tmem + col_o(h), tmem + col_s(h) + k * 8, dv + uint64_t(k) * 128u, kIdescPV,
                   (first && k == 0) ? 0u : 1u);
          if (++vs == kVStages) { vs = 0; vph ^= 1; }
          return true;
        };
        // S_h = Q K^T for the stream's next block.
        auto issue_s = [&](int h) -> bool {
          if (!mbar_wait(&bars->k_full[ks], kph, abort, a.wait_cycles)) return false;
          const uint64_t dk = dk0 + uint64_t(ks * kStageDesc);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            // step k of the 128-deep contraction: 32 bytes along a 128-byte
            // swizzled row, then the second 64-column region
            const uint64_t off = uint64_t((k >> 2) * (kRegionBytes >> 4) + (k & 3) * 2);
            mma_ss(tmem + col_s(h), dq + off, dk + off, kIdescQK, k > 0 ? 1u : 0u);
          }
          if (withhold && h == 0) withhold = false;
          else mma_commit(&bars->s_full[h]);
          if (++ks == kKStages) { ks = 0; kph ^= 1; }
          return true;
        };
#endif
        if (!(ok = mbar_wait(&bars->q_full, uc & 1, abort, a.wait_cycles))) break;
        // Order per step j: PV_0(j-1), S_0(j), PV_1(j-1), S_1(j) -- the load
        // order of K and of V.  Where stream 1 has one block fewer, its last
        // PV comes right after S_0 of the extra block, again in load order.
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
        mma_commit(&bars->q_empty);  // every S of this unit issued
        if (!(ok = issue_pv(0, t.nb0 == 1))) break;
        if (t.nb1 == t.nb0 && t.nb1 > 0 && !(ok = issue_pv(1, t.nb1 == 1))) break;
        mma_commit(&bars->o_ready);
      }
      // Every MMA issued here completes before TMEM is released.
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
    uint32_t use = 0, base = 0, uc = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < a.n_tiles; tile += gridDim.x, ++uc) {
      const Unit t = decode(a, tile);
      const int mine = h ? t.nb1 : t.nb0;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < mine; ++j, ++use) {
        const int b = block_of(t, h, j);
        const bool inA = b < t.nbA;
        const int64_t rows_left = (inA ? t.nA : a.Lq) - int64_t(inA ? b : b - t.nbA) * 128;
        const int nv = rows_left < 128 ? int(rows_left) : 128;  // valid keys of the block
        if (!(ok = warp_wait(&bars->s_full[h], use & 1, abort, a.wait_cycles))) break;
        tc_fence_after();
        if (row == 0) {
          // S_h(j) is complete, and with it every MMA issued before it: the K
          // stage it read and the V stage of this stream's previous PV are free.
          mbar_arrive(&bars->k_empty[(base + uint32_t(seq_pos(t, h, j))) % kKStages]);
          if (j > 0) mbar_arrive(&bars->v_empty[(base + uint32_t(seq_pos(t, h, j - 1))) % kVStages]);
        }
        uint32_t sr[128];  // raw fp32 logits of this row
#define SV(i) __uint_as_float(sr[i])
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        tmem_ld_wait();
        if (nv < 128) {  // ragged block: columns past the valid keys never count
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i >= nv) sr[i] = 0xff800000u;  // -inf
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
        const float m_new = fmaxf(m, bmax * a.sl2);  // scale > 0
        if (j == 0) {
          m = m_new;
        } else if (__any_sync(0xffffffffu, m_new > m + kRescaleLog2)) {
          // S_h of this block is complete, so the PV before it into O_h is too.
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
        float2 acc[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[k] = make_float2(0.f, 0.f);
        const float2 sl2x2 = make_float2(a.sl2, a.sl2), negm2 = make_float2(-m, -m);
        // P in two halves of 64 columns (32 packed TMEM columns each); P
        // overwrites S columns whose values are already in registers.
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int c = 64 * hh + 2 * i;
            const float2 e = ffma2(make_float2(SV(c), SV(c + 1)), sl2x2, negm2);
            const float2 p = (FKV_POLY_EVERY > 0 && i % (FKV_POLY_EVERY > 0 ? FKV_POLY_EVERY : 1) ==
                                                       (FKV_POLY_EVERY > 0 ? FKV_POLY_EVERY : 1) - 1)
                                 ? exp2_poly2(e)
                                 : make_float2(ex2(e.x), ex2(e.y));
            acc[i & 3] = fadd2(acc[i & 3], p);
            pk[i] = pack_bf16(p.x, p.y);
          }
          tmem_st32(tS + 32 * hh, pk);
        }
#undef SV
        const float2 s2 = fadd2(fadd2(acc[0], acc[1]), fadd2(acc[2], acc[3]));
        l += s2.x + s2.y;
        tmem_st_wait();
        if (nv < 128) {
          // V rows past the valid keys may hold anything (P is 0 there, but
          // 0 * NaN is not 0): zero them before the PV MMA reads the stage.
          const uint32_t pos = base + uint32_t(seq_pos(t, h, j));
          const uint32_t s = pos % kVStages, u = pos / kVStages;
          if (!(ok = warp_wait(&bars->v_full[s], u & 1, abort, a.wait_cycles))) break;
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
        mbar_arrive(&bars->p_full[h]);
      }
      if (!ok) break;
      // V stage of this stream's last PV (released once both PV chains are done)
      const uint32_t last_v = mine > 0 ? (base + uint32_t(seq_pos(t, h, mine - 1))) % kVStages : 0u;
      base += uint32_t(t.nb);
      // ---- merge the two streams and write this thread's 64 output columns
      if (!(ok = warp_wait(&bars->o_ready, uc & 1, abort, a.wait_cycles))) break;
      tc_fence_after();
      if (row == 0 && mine > 0) mbar_arrive(&bars->v_empty[last_v]);
      if (!(ok = warp_wait(&bars->x_read, (uc & 1) ^ 1, abort, a.wait_cycles))) break;  // last unit's reads done
      bars->xml[h][row] = make_float2(m, l);
      mbar_arrive(&bars->x_full);
      if (!(ok = warp_wait(&bars->x_full, uc & 1, abort, a.wait_cycles))) break;
      const float2 other = bars->xml[h ^ 1][row];
      mbar_arrive(&bars->x_read);
      const float m0 = h ? other.x : m, l0 = h ? other.y : l;
      const float m1 = h ? m : other.x, l1 = h ? l : other.y;
      const bool two = t.nb1 > 0;
      const float M = two ? fmaxf(m0, m1) : m0;
      const float a0 = ex2(m0 - M), a1 = two ? ex2(m1 - M) : 0.f;
      const float inv = 1.f / (l0 * a0 + (two ? l1 * a1 : 0.f));
      const float c0 = a0 * inv, c1 = a1 * inv;
      // 64 columns per thread, merged and written 32 at a time.
      const int64_t q = int64_t(t.qt) * 128 + row;
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

// Evaluates the attention kernel's FMA-pipe exp2 on an array (for testing it
// against the hardware exp2 and its error bound).
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int64_t n) {
  const int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  if (i + 1 < n) {
    const float2 r = exp2_poly2(make_float2(x[i], x[i + 1]));
    y[i] = r.x;
    y[i + 1] = r.y;
  } else if (i < n) {
    y[i] = exp2_poly2(make_float2(x[i], 0.f)).x;
  }
}

}  // namespace sm100


cudaError_t launch_attend_sm100(const Dims& d, const void* q_cur, const void* k_cur,
                                const void* v_cur, const void* k_comp, const void* v_comp,
                                const int32_t* kept_cnt, void* out, int32_t* status,
                                cudaStream_t s, long long wait_cycles, bool withhold_s0) {
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
  a.wait_cycles = wait_cycles;
  a.withhold_s0 = withhold_s0 ? 1 : 0;
  cudaError_t e = cudaFuncSetAttribute(attend_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(kAttnSmem));
  if (e != cudaSuccess) return e;
  const int grid = a.n_tiles < num_sms() ? a.n_tiles : num_sms();
  return launch_kernel(attend_sm100_kernel, dim3(grid), dim3(kAttnThreads), kAttnSmem, s, d.pdl,
                       tq, tkc, tvc, tkn, tvn, a);
}

cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  sm100::exp2_poly_kernel<<<unsigned((pairs + 255) / 256), 256, 0, s>>>(x, y, n);
  return cudaGetLastError();
}

}  // namespace fkv
