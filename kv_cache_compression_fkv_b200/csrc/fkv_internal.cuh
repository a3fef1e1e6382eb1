// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fkv.h"

namespace fkv {

// Resolved sizes of one call, derived once from fkv_params_t on the host.
struct Dims {
  int L, H, D, T, F, Fc;
  int LH;            // L * H
  int64_t N;         // history tokens per head, F * T
  int64_t Lq;        // chunk queries per head, Fc * T
  int stride;        // frame mode scoring stride
  int64_t n_s;       // frame mode: scoring queries per head
  int64_t n_score_q; // token mode: q_score rows per head
  int64_t S, R;      // token mode sink / recent tokens
  int64_t nseg;      // scored segments per head (F, or N - S - R)
  int64_t max_kept;  // kept_idx entries per head (F, or N)
  int64_t seg_len;   // rows per segment (T, or 1)
  int64_t comp_rows; // rows per head of the compressed cache
  float scale;
  bool bf16;
  bool token;
  bool score_with_chunk;  // frame mode: chunk keys in the scoring normaliser
  bool static_token_mask; // frame mode: per-token static masks, kept lists in tokens
  int elem;          // bytes per activation element
  bool pdl = false;  // launch as a programmatic dependent of the previous kernel
};

// Layout of the frame-mode partial softmax statistics (part_ml, float2
// (max, sum), [head][scoring row][entry], a row's entries contiguous): per
// head and row, F*split frame entries
// (entry f*split + i is the i-th piece of frame f), then `chunk` entries for
// the chunk's own keys when they join the normaliser; E entries per head.
//   tensor-core scoring (bf16): one entry per 128-key block, split =
//     ceil(T/128), chunk = ceil(Lq/128) or 0, E = F*split + chunk;
//   CUDA-core scoring (fp32): one entry per frame, split = 1, chunk = 1 or 0,
//     E = F + 1.
struct ScoreLayout {
  int split, chunk, E;
};
inline ScoreLayout score_layout(const Dims& d) {
  ScoreLayout s;
  if (d.bf16) {
    s.split = (d.T + 127) / 128;
    s.chunk = d.score_with_chunk ? int((d.Lq + 127) / 128) : 0;
    s.E = d.F * s.split + s.chunk;
  } else {
    s.split = 1;
    s.chunk = d.score_with_chunk ? 1 : 0;
    s.E = d.F + 1;
  }
  return s;
}

// Workspace layout (byte offsets from the workspace base, 256-B aligned).
struct WsLayout {
  size_t status;     // int32[2]: first device error, detail
  size_t part_ml;    // frame mode: float2 [LH][n_s][E] (max, sum) per entry, the
                     // layout of score_layout()
  size_t row_ml;     // frame mode: float2 [LH][n_s] per-row (max, sum)
  size_t qbar;       // token mode: float [LH][D] summed scoring queries
  size_t total;
};

WsLayout ws_layout(const Dims& d);


// Programmatic dependent launch.  Inside one call sequence (fkv_step), every
// kernel after the first is launched so that the launch is prepared while its
// predecessor on the stream is still running and its CTAs start as soon as
// that grid has finished; it runs its on-chip prologue (shared-memory
// barriers, tensor memory, tensor-map prefetch), then pdl_wait() blocks until
// the predecessor grid has completed and its memory is visible -- before the
// kernel reads or writes any global memory.  No kernel signals its
// dependents early (griddepcontrol.launch_dependents): measured, dependents
// resident while their predecessor still runs slowed it down more than the
// early start saved.  Launched without the attribute, pdl_wait() returns at
// once.
#ifndef FKV_PDL
#define FKV_PDL 1
#endif
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches `kernel`, as a programmatic dependent of the previous work on `s`
// when `pdl` is set.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                 cudaStream_t s, bool pdl, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (pdl && FKV_PDL) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Records the first device-side error of a call sequence.
__device__ __forceinline__ void report(int32_t* status, int32_t code, int32_t detail) {
  if (atomicCAS(status, 0, code) == 0) atomicExch(status + 1, detail);
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Order-preserving map of a float to uint32 (larger float -> larger key);
// -0.0 is folded onto +0.0 so the two compare equal, as in IEEE comparison.
__device__ __forceinline__ uint32_t ordered_key(float x) {
  uint32_t b = __float_as_uint(x);
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// ---- launchers (each returns cudaGetLastError() of its launches) ----------
cudaError_t launch_score_frame_simt(const Dims& d, const void* q_cur, const void* k_hist,
                                    const void* k_cur, const uint8_t* head_role, float2* part_ml,
                                    cudaStream_t s);
// part_ml has the layout of score_layout(d), [head][n_s rows][E entries]; the
// finalize overwrites the m of each frame's first entry with that frame's
// per-row mass.  poison (nullable): a status word; when it is nonzero at the
// finalize, every dynamic head's scores are written NaN.
cudaError_t launch_score_frame_finalize(const Dims& d, const ScoreLayout& sl,
                                        const uint8_t* head_role, float2* part_ml,
                                        float2* row_ml, float* seg_score, cudaStream_t s,
                                        const int32_t* poison = nullptr);
// fkv_score_segments after its host-side checks; poison_on_error: scores of
// dynamic heads come out NaN when the workspace status word is nonzero by the
// time the scores are summed (used where the caller cannot read the status).
int32_t score_segments_checked(const fkv_params_t* p, const void* q_cur, const void* q_score,
                               const void* k_hist, const void* k_cur, const uint8_t* head_role,
                               float* seg_score, void* ws, void* stream, bool poison_on_error);
cudaError_t launch_score_token(const Dims& d, const void* q_score, const void* k_hist,
                               float* qbar, float* seg_score, cudaStream_t s);
cudaError_t launch_select_frame(const Dims& d, const float* seg_score, const uint8_t* head_role,
                                const uint8_t* static_mask, const int32_t* k_per_head,
                                int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                cudaStream_t s);
cudaError_t launch_select_frame_tokens(const Dims& d, const float* seg_score,
                                       const uint8_t* head_role, const uint8_t* static_mask,
                                       const int32_t* k_per_head, int32_t* kept_idx,
                                       int32_t* kept_cnt, int32_t* status, cudaStream_t s);
cudaError_t launch_select_token(const Dims& d, const float* seg_score, const int32_t* k_per_head,
                                int32_t* kept_idx, int32_t* kept_cnt, int32_t* status,
                                cudaStream_t s);
cudaError_t launch_gather(const Dims& d, const void* k_hist, const void* v_hist,
                          const int32_t* kept_idx, const int32_t* kept_cnt, void* k_comp,
                          void* v_comp, int32_t* status, cudaStream_t s);
cudaError_t launch_score_frame_sm100(const Dims& d, const void* q_cur, const void* k_hist,
                                     const void* k_cur, const uint8_t* head_role, float2* part_ml,
                                     int32_t* status, cudaStream_t s);
// wait_cycles bounds every mbarrier wait; withhold_s0 (diagnostic) makes CTA 0
// withhold one completion signal so that a wait runs out.
constexpr long long kProductionWaitCycles = 2000000000LL;
cudaError_t launch_attend_sm100(const Dims& d, const void* q_cur, const void* k_cur,
                                const void* v_cur, const void* k_comp, const void* v_comp,
                                const int32_t* kept_cnt, void* out, int32_t* status,
                                cudaStream_t s, long long wait_cycles = kProductionWaitCycles,
                                bool withhold_s0 = false);
cudaError_t launch_gather_rope(const Dims& d, const void* k_hist, const void* v_hist,
                               const int32_t* kept_idx, const int32_t* kept_cnt,
                               const float* omega, int32_t n_pairs, void* k_comp, void* v_comp,
                               int32_t* status, cudaStream_t s);
cudaError_t launch_advance(const Dims& d, int64_t out_segments, const void* k_comp,
                           const void* v_comp, const int32_t* kept_cnt, const void* k_cur,
                           const void* v_cur, void* k_next, void* v_next, int32_t* status,
                           cudaStream_t s);
cudaError_t launch_exp2_poly(const float* x, float* y, int64_t n, cudaStream_t s);
// Hardware-rate diagnostics (diag.cu): cycles of n tcgen05.mma of one shape
// issued back to back by one thread, and of n ex2 per warp.
cudaError_t launch_diag_mma_rate(int shape, int n, int busy, long long* cycles, int32_t* status,
                                 cudaStream_t s);
cudaError_t launch_diag_ex2_rate(int n, int warps, long long* cycles, cudaStream_t s);
// e4m3 quantisation (quant_fp8.cu): the kept history segments into the
// compressed cache, the chunk's segments and query rows, or all three in one
// launch (the fp8 step).
cudaError_t launch_quant_kept(const Dims& d, const int32_t* kept_idx, const int32_t* kept_cnt,
                              const void* k_hist, const void* v_hist, const fkv_fp8_cache_t& c,
                              int32_t* status, cudaStream_t s);
cudaError_t launch_quant_chunk(const Dims& d, const void* q_cur, const void* k_cur,
                               const void* v_cur, const fkv_fp8_cache_t& c, int32_t* status,
                               cudaStream_t s);
cudaError_t launch_quant_step(const Dims& d, const int32_t* kept_idx, const int32_t* kept_cnt,
                              const void* k_hist, const void* v_hist, const void* q_cur,
                              const void* k_cur, const void* v_cur, const fkv_fp8_cache_t& c,
                              int32_t* status, cudaStream_t s);
cudaError_t launch_attend_fp8_sm100(const Dims& d, const fkv_fp8_cache_t& c,
                                    const int32_t* kept_cnt, void* out, int32_t* status,
                                    cudaStream_t s);
// Comparison selectors (uniform eviction / random drop) of every head.
cudaError_t launch_heuristic(const Dims& d, int32_t policy, uint64_t seed,
                             const int32_t* k_per_head, float* seg_score, int32_t* kept_idx,
                             int32_t* kept_cnt, int32_t* status, cudaStream_t s);
cudaError_t launch_attend_simt(const Dims& d, const void* q_cur, const void* k_cur,
                               const void* v_cur, const void* k_comp, const void* v_comp,
                               const int32_t* kept_cnt, void* out, cudaStream_t s);

// SM count of the current device (cached per device; 148 if unknown).
int num_sms();

}  // namespace fkv
