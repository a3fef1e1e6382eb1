// Host side of the C ABI: argument validation, workspace layout and the
// launch order of the chunk step.  Every check that can be done without
// device data runs before the first launch.
#include <stdio.h>

#include "fkv_internal.cuh"

namespace fkv {

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const Dims& d) {
  WsLayout w{};
  size_t off = 0;
  w.status = off;
  off += 256;
  w.part_ml = w.row_ml = w.qbar = off;
  if (!d.token) {
    w.part_ml = off;
    off = align256(off + sizeof(float2) * size_t(d.LH) * size_t(score_layout(d).E) *
                             size_t(d.n_s));
    w.row_ml = off;
    off = align256(off + sizeof(float2) * size_t(d.LH) * size_t(d.n_s));
  } else {
    w.qbar = off;
    off = align256(off + sizeof(float) * size_t(d.LH) * size_t(d.D));
  }
  w.total = off;
  return w;
}

// Largest sizes accepted; they keep every index computation inside int64 and
// grid dimensions inside CUDA limits.
static const int64_t kMaxRowsPerHead = int64_t(1) << 26;
static const int kMaxFrames = 1024;
static const int kMaxHeadsTotal = 65535;

static int32_t make_dims(const fkv_params_t* p, Dims* d) {
  if (!p) return FKV_ERR_INVALID_ARG;
  if (p->dtype != FKV_DTYPE_BF16 && p->dtype != FKV_DTYPE_FP32) return FKV_ERR_INVALID_ARG;
  if (p->granularity != FKV_GRAN_FRAME && p->granularity != FKV_GRAN_TOKEN)
    return FKV_ERR_INVALID_ARG;
  if (p->num_layers < 1 || p->num_heads < 1 || p->frame_tokens < 1 || p->hist_frames < 0 ||
      p->chunk_frames < 1 || p->comp_rows < 0)
    return FKV_ERR_SHAPE;
  if (!(p->scale > 0.f) || p->scale > 3.0e38f) return FKV_ERR_INVALID_ARG;  // finite, > 0
  d->L = p->num_layers;
  d->H = p->num_heads;
  d->D = p->head_dim;
  d->T = p->frame_tokens;
  d->F = p->hist_frames;
  d->Fc = p->chunk_frames;
  if (int64_t(d->L) * d->H > kMaxHeadsTotal) return FKV_ERR_SHAPE;
  d->LH = d->L * d->H;
  d->N = int64_t(d->F) * d->T;
  d->Lq = int64_t(d->Fc) * d->T;
  if (d->N > kMaxRowsPerHead || d->Lq > kMaxRowsPerHead || p->comp_rows > kMaxRowsPerHead)
    return FKV_ERR_SHAPE;
  d->bf16 = p->dtype == FKV_DTYPE_BF16;
  d->token = p->granularity == FKV_GRAN_TOKEN;
  if (p->flags & ~int32_t(FKV_FLAG_SCORE_WITH_CHUNK | FKV_FLAG_STATIC_TOKEN_MASK))
    return FKV_ERR_INVALID_ARG;
  d->score_with_chunk = (p->flags & FKV_FLAG_SCORE_WITH_CHUNK) != 0;
  d->static_token_mask = (p->flags & FKV_FLAG_STATIC_TOKEN_MASK) != 0;
  if (d->token && (d->score_with_chunk || d->static_token_mask))
    return FKV_ERR_UNSUPPORTED;  // frame-mode options
  d->elem = d->bf16 ? 2 : 4;
  if (d->bf16) {
    if (d->D != 128) return FKV_ERR_UNSUPPORTED;
  } else {
    if (d->D < 4 || d->D > 128 || d->D % 4 != 0) return FKV_ERR_UNSUPPORTED;
  }
  d->scale = p->scale;
  d->comp_rows = p->comp_rows;
  d->stride = 1;
  d->n_s = 0;
  d->n_score_q = 0;
  d->S = d->R = 0;
  if (!d->token) {
    if (d->F > kMaxFrames) return FKV_ERR_SHAPE;
    if (p->score_stride < 1) return FKV_ERR_SHAPE;
    d->stride = p->score_stride;
    d->n_s = (d->Lq + d->stride - 1) / d->stride;
    d->nseg = d->F;
    d->max_kept = d->static_token_mask ? d->N : d->F;
    d->seg_len = d->static_token_mask ? 1 : d->T;
  } else {
    if (p->sink_tokens < 0 || p->recent_tokens < 0) return FKV_ERR_SHAPE;
    d->S = p->sink_tokens;
    d->R = p->recent_tokens;
    if (d->S + d->R > d->N) return FKV_ERR_SHAPE;
    d->nseg = d->N - d->S - d->R;
    if (d->nseg > 0 && p->n_score_q < 1) return FKV_ERR_SHAPE;
    d->n_score_q = p->n_score_q < 0 ? 0 : p->n_score_q;
    d->max_kept = d->N;
    d->seg_len = 1;
  }
  return FKV_OK;
}

static bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

static int32_t check_ws(const Dims& d, void* ws) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FKV_ERR_WORKSPACE;
  (void)d;
  return FKV_OK;
}

static int32_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return FKV_OK;
  fprintf(stderr, "fkv: CUDA error %d (%s)\n", int(e), cudaGetErrorString(e));
  return FKV_ERR_CUDA;
}

static int32_t* status_ptr(void* ws) { return reinterpret_cast<int32_t*>(ws); }
static char* ws_at(void* ws, size_t off) { return reinterpret_cast<char*>(ws) + off; }

// ---- the five steps, after validation -------------------------------------

static int32_t do_score(const Dims& d, const void* q_cur, const void* q_score, const void* k_hist,
                        const void* k_cur, const uint8_t* head_role, float* seg_score, void* ws,
                        cudaStream_t s, bool poison_on_error = false) {
  WsLayout w = ws_layout(d);
  if (d.token) {
    if (d.nseg == 0) return FKV_OK;
    return cuda_status(launch_score_token(d, q_score, k_hist,
                                          reinterpret_cast<float*>(ws_at(ws, w.qbar)), seg_score,
                                          s));
  }
  if (d.F == 0) return FKV_OK;
  float2* part = reinterpret_cast<float2*>(ws_at(ws, w.part_ml));
  float2* rows = reinterpret_cast<float2*>(ws_at(ws, w.row_ml));
  // bf16: tensor-core scoring; fp32: CUDA-core scoring (fp32 accuracy mode).
  cudaError_t e = d.bf16 ? launch_score_frame_sm100(d, q_cur, k_hist, k_cur, head_role, part,
                                                    status_ptr(ws), s)
                         : launch_score_frame_simt(d, q_cur, k_hist, k_cur, head_role, part, s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(launch_score_frame_finalize(d, score_layout(d), head_role, part, rows,
                                                 seg_score, s,
                                                 poison_on_error ? status_ptr(ws) : nullptr));
}

static int32_t do_select(const Dims& d, const float* seg_score, const uint8_t* head_role,
                         const uint8_t* static_mask, const int32_t* k_per_head, int32_t* kept_idx,
                         int32_t* kept_cnt, void* ws, cudaStream_t s) {
  if (d.token)
    return cuda_status(
        launch_select_token(d, seg_score, k_per_head, kept_idx, kept_cnt, status_ptr(ws), s));
  if (d.static_token_mask)
    return cuda_status(launch_select_frame_tokens(d, seg_score, head_role, static_mask, k_per_head,
                                                  kept_idx, kept_cnt, status_ptr(ws), s));
  return cuda_status(launch_select_frame(d, seg_score, head_role, static_mask, k_per_head,
                                         kept_idx, kept_cnt, status_ptr(ws), s));
}

static int32_t do_gather(const Dims& d, const void* k_hist, const void* v_hist,
                         const int32_t* kept_idx, const int32_t* kept_cnt, void* k_comp,
                         void* v_comp, void* ws, cudaStream_t s) {
  return cuda_status(
      launch_gather(d, k_hist, v_hist, kept_idx, kept_cnt, k_comp, v_comp, status_ptr(ws), s));
}

static int32_t do_attend(const Dims& d, const void* q_cur, const void* k_cur, const void* v_cur,
                         const void* k_comp, const void* v_comp, const int32_t* kept_cnt,
                         void* out, void* ws, cudaStream_t s) {
  // bf16: tensor-core attention; fp32: CUDA-core attention (fp32 accuracy mode).
  if (d.bf16)
    return cuda_status(launch_attend_sm100(d, q_cur, k_cur, v_cur, k_comp, v_comp, kept_cnt, out,
                                           status_ptr(ws), s));
  return cuda_status(launch_attend_simt(d, q_cur, k_cur, v_cur, k_comp, v_comp, kept_cnt, out, s));
}

// Kernel launches of one fkv_step; must follow the do_* functions above.
static int32_t step_launch_count(const Dims& d) {
  int32_t n = 0;
  if (d.token) n += d.nseg > 0 ? 2 : 0;   // q-sum, phi
  else n += d.F > 0 ? 3 : 0;              // partial statistics, row merge, frame masses
  n += 1;                                 // select
  n += 1;                                 // gather
  n += 1;                                 // attention
  return n;
}

}  // namespace fkv

using namespace fkv;

extern "C" {

const char* fkv_status_string(int32_t status) {
  switch (status) {
    case FKV_OK: return "FKV_OK";
    case FKV_ERR_INVALID_ARG: return "FKV_ERR_INVALID_ARG: null pointer, bad enum or misaligned pointer";
    case FKV_ERR_SHAPE: return "FKV_ERR_SHAPE: sizes negative, inconsistent or above limits";
    case FKV_ERR_UNSUPPORTED: return "FKV_ERR_UNSUPPORTED: request not implemented by this build";
    case FKV_ERR_CUDA: return "FKV_ERR_CUDA: a CUDA call or launch failed";
    case FKV_ERR_TIMEOUT: return "FKV_ERR_TIMEOUT: a bounded device wait gave up";
    case FKV_ERR_WORKSPACE: return "FKV_ERR_WORKSPACE: workspace null, too small or misaligned";
    case FKV_ERR_DEVICE_ARG: return "FKV_ERR_DEVICE_ARG: device-side argument out of range";
    default: return "FKV_ERR_UNKNOWN";
  }
}

int32_t fkv_abi_version(void) { return FKV_ABI_VERSION; }

int32_t fkv_check_params(const fkv_params_t* p) {
  Dims d;
  return make_dims(p, &d);
}

int32_t fkv_num_segments(const fkv_params_t* p, int64_t* nseg) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!nseg) return FKV_ERR_INVALID_ARG;
  *nseg = d.nseg;
  return FKV_OK;
}

int32_t fkv_max_kept(const fkv_params_t* p, int64_t* max_kept) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!max_kept) return FKV_ERR_INVALID_ARG;
  *max_kept = d.max_kept;
  return FKV_OK;
}

int32_t fkv_max_comp_rows(const fkv_params_t* p, int64_t* rows) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!rows) return FKV_ERR_INVALID_ARG;
  *rows = d.N;
  return FKV_OK;
}

int32_t fkv_workspace_size(const fkv_params_t* p, size_t* bytes) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!bytes) return FKV_ERR_INVALID_ARG;
  *bytes = ws_layout(d).total;
  return FKV_OK;
}

int32_t fkv_step_launches(const fkv_params_t* p, int32_t* launches) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!launches) return FKV_ERR_INVALID_ARG;
  *launches = step_launch_count(d);
  return FKV_OK;
}

int32_t fkv_exp2_emulated(const float* x, float* y, int64_t n, void* stream) {
  if (n < 0) return FKV_ERR_SHAPE;
  if (n > 0 && (!x || !y)) return FKV_ERR_INVALID_ARG;
  return cuda_status(launch_exp2_poly(x, y, n, static_cast<cudaStream_t>(stream)));
}

int32_t fkv_diag_mma_rate(int32_t shape, int32_t n_mma, int32_t busy, int64_t* cycles, void* ws,
                          void* stream) {
  if (shape < 0 || shape > 10 || n_mma < 8 || n_mma > 4096 || n_mma % 8 != 0)
    return FKV_ERR_SHAPE;
  if (!cycles) return FKV_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FKV_ERR_WORKSPACE;
  return cuda_status(launch_diag_mma_rate(shape, n_mma, busy != 0 ? 1 : 0,
                                          reinterpret_cast<long long*>(cycles), status_ptr(ws),
                                          static_cast<cudaStream_t>(stream)));
}

int32_t fkv_diag_ex2_rate(int32_t n, int32_t warps, int64_t* cycles, void* stream) {
  if (n < 8 || n > (1 << 20) || n % 8 != 0 || warps < 1 || warps > 4) return FKV_ERR_SHAPE;
  if (!cycles) return FKV_ERR_INVALID_ARG;
  return cuda_status(launch_diag_ex2_rate(n, warps, reinterpret_cast<long long*>(cycles),
                                          static_cast<cudaStream_t>(stream)));
}

int32_t fkv_workspace_init(void* ws, size_t bytes, void* stream) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || bytes < 256) return FKV_ERR_WORKSPACE;
  return cuda_status(cudaMemsetAsync(ws, 0, bytes, static_cast<cudaStream_t>(stream)));
}

int32_t fkv_read_status(const void* ws, void* stream, int32_t* device_status, int32_t* detail) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return FKV_ERR_WORKSPACE;
  int32_t h[2] = {0, -1};
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (device_status) *device_status = h[0];
  if (detail) *detail = h[0] == 0 ? -1 : h[1];
  return FKV_OK;
}

int32_t fkv_score_segments(const fkv_params_t* p, const void* q_cur, const void* q_score,
                           const void* k_hist, const void* k_cur, const uint8_t* head_role,
                           float* seg_score, void* ws, void* stream) {
  return fkv::score_segments_checked(p, q_cur, q_score, k_hist, k_cur, head_role, seg_score, ws,
                                     stream, false);
}

}  // extern "C"

int32_t fkv::score_segments_checked(const fkv_params_t* p, const void* q_cur,
                                    const void* q_score, const void* k_hist, const void* k_cur,
                                    const uint8_t* head_role, float* seg_score, void* ws,
                                    void* stream, bool poison_on_error) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if ((!k_hist && d.N > 0) || (!seg_score && d.nseg > 0)) return FKV_ERR_INVALID_ARG;
  if (d.token) {
    if (!q_score && d.nseg > 0) return FKV_ERR_INVALID_ARG;
    if (!aligned16(q_score)) return FKV_ERR_INVALID_ARG;
  } else {
    if (!q_cur || !head_role) return FKV_ERR_INVALID_ARG;
    if (!aligned16(q_cur)) return FKV_ERR_INVALID_ARG;
  }
  if (!aligned16(k_hist)) return FKV_ERR_INVALID_ARG;
  if (d.score_with_chunk && (!k_cur || !aligned16(k_cur))) return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return do_score(d, q_cur, q_score, k_hist, k_cur, head_role, seg_score, ws,
                  static_cast<cudaStream_t>(stream), poison_on_error);
}

extern "C" {

int32_t fkv_select_topk(const fkv_params_t* p, const float* seg_score, const uint8_t* head_role,
                        const uint8_t* static_mask, const int32_t* k_per_head, int32_t* kept_idx,
                        int32_t* kept_cnt, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if ((!seg_score && d.nseg > 0) || !k_per_head || (!kept_idx && d.max_kept > 0) || !kept_cnt)
    return FKV_ERR_INVALID_ARG;
  if (!d.token && (!head_role || (!static_mask && d.F > 0))) return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return do_select(d, seg_score, head_role, static_mask, k_per_head, kept_idx, kept_cnt, ws,
                   static_cast<cudaStream_t>(stream));
}

int32_t fkv_compact_gather(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                           const int32_t* kept_idx, const int32_t* kept_cnt, void* k_comp,
                           void* v_comp, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (((!k_hist || !v_hist) && d.N > 0) || (!kept_idx && d.max_kept > 0) || !kept_cnt ||
      ((!k_comp || !v_comp) && d.comp_rows > 0))
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(k_hist) || !aligned16(v_hist) || !aligned16(k_comp) || !aligned16(v_comp))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return do_gather(d, k_hist, v_hist, kept_idx, kept_cnt, k_comp, v_comp, ws,
                   static_cast<cudaStream_t>(stream));
}

int32_t fkv_attend_compressed(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                              const void* v_cur, const void* k_comp, const void* v_comp,
                              const int32_t* kept_cnt, void* out, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!q_cur || !k_cur || !v_cur || ((!k_comp || !v_comp) && d.comp_rows > 0) || !kept_cnt || !out)
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(q_cur) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(k_comp) ||
      !aligned16(v_comp) || !aligned16(out))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return do_attend(d, q_cur, k_cur, v_cur, k_comp, v_comp, kept_cnt, out, ws,
                   static_cast<cudaStream_t>(stream));
}

int32_t fkv_diag_attend_timeout(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                                const void* v_cur, const void* k_comp, const void* v_comp,
                                const int32_t* kept_cnt, void* out, int64_t wait_cycles, void* ws,
                                void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!d.bf16) return FKV_ERR_UNSUPPORTED;  // the tensor-core kernel's waits
  if (wait_cycles < 10000 || wait_cycles > kProductionWaitCycles) return FKV_ERR_SHAPE;
  if (!q_cur || !k_cur || !v_cur || ((!k_comp || !v_comp) && d.comp_rows > 0) || !kept_cnt || !out)
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(q_cur) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(k_comp) ||
      !aligned16(v_comp) || !aligned16(out))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return cuda_status(launch_attend_sm100(d, q_cur, k_cur, v_cur, k_comp, v_comp, kept_cnt, out,
                                         status_ptr(ws), static_cast<cudaStream_t>(stream),
                                         wait_cycles, true));
}

int32_t fkv_compact_gather_rope(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                                const int32_t* kept_idx, const int32_t* kept_cnt,
                                const float* omega, int32_t n_pairs, void* k_comp, void* v_comp,
                                void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (d.token || d.static_token_mask) return FKV_ERR_UNSUPPORTED;  // frames only
  if (n_pairs < 0 || 2 * n_pairs > d.D) return FKV_ERR_SHAPE;
  if (((!k_hist || !v_hist) && d.N > 0) || (!kept_idx && d.max_kept > 0) || !kept_cnt ||
      ((!k_comp || !v_comp) && d.comp_rows > 0) || (n_pairs > 0 && !omega))
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(k_hist) || !aligned16(v_hist) || !aligned16(k_comp) || !aligned16(v_comp))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return cuda_status(launch_gather_rope(d, k_hist, v_hist, kept_idx, kept_cnt, omega, n_pairs,
                                        k_comp, v_comp, status_ptr(ws),
                                        static_cast<cudaStream_t>(stream)));
}

int32_t fkv_cache_advance(const fkv_params_t* p, const void* k_comp, const void* v_comp,
                          const int32_t* kept_cnt, const void* k_cur, const void* v_cur,
                          int64_t out_segments, void* k_next, void* v_next, void* ws,
                          void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  const int64_t chunk_segs = d.Lq / d.seg_len;
  if (out_segments < chunk_segs || out_segments > d.max_kept + chunk_segs ||
      out_segments * d.seg_len > kMaxRowsPerHead)
    return FKV_ERR_SHAPE;
  const bool old = out_segments > chunk_segs;
  if ((old && (!k_comp || !v_comp)) || !kept_cnt || !k_cur || !v_cur || !k_next || !v_next)
    return FKV_ERR_INVALID_ARG;
  const void* ptrs[] = {k_cur, v_cur, k_next, v_next};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FKV_ERR_INVALID_ARG;
  if (old && (!aligned16(k_comp) || !aligned16(v_comp))) return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return cuda_status(launch_advance(d, out_segments, k_comp, v_comp, kept_cnt, k_cur, v_cur,
                                    k_next, v_next, status_ptr(ws),
                                    static_cast<cudaStream_t>(stream)));
}

int32_t fkv_step(const fkv_params_t* p, const fkv_step_io_t* io, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!io) return FKV_ERR_INVALID_ARG;
  if (!io->q_cur || !io->k_cur || !io->v_cur || ((!io->k_hist || !io->v_hist) && d.N > 0) ||
      !io->k_per_head || (!io->seg_score && d.nseg > 0) || (!io->kept_idx && d.max_kept > 0) ||
      !io->kept_cnt || ((!io->k_comp || !io->v_comp) && d.comp_rows > 0) || !io->out)
    return FKV_ERR_INVALID_ARG;
  if (d.token ? (!io->q_score && d.nseg > 0) : (!io->head_role || (!io->static_mask && d.F > 0)))
    return FKV_ERR_INVALID_ARG;
  const void* ptrs[] = {io->q_cur, io->k_cur, io->v_cur, io->k_hist, io->v_hist,
                        io->k_comp, io->v_comp, io->out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FKV_ERR_INVALID_ARG;
  if (d.token && !aligned16(io->q_score)) return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = do_score(d, io->q_cur, io->q_score, io->k_hist, io->k_cur, io->head_role,
                     io->seg_score, ws, s)))
    return st;
  // Every kernel after the scoring follows one of this call's own kernels on
  // the stream: launch it as a programmatic dependent (its on-chip prologue
  // overlaps the previous kernel's tail; it waits for that grid before it
  // touches global memory).  Without scoring work the select kernel is the
  // first of the call and launches normally.
  Dims dp = d;
  dp.pdl = d.token ? d.nseg > 0 : d.F > 0;
  if ((st = do_select(dp, io->seg_score, io->head_role, io->static_mask, io->k_per_head,
                      io->kept_idx, io->kept_cnt, ws, s)))
    return st;
  dp.pdl = true;
  if ((st = do_gather(dp, io->k_hist, io->v_hist, io->kept_idx, io->kept_cnt, io->k_comp,
                      io->v_comp, ws, s)))
    return st;
  return do_attend(dp, io->q_cur, io->k_cur, io->v_cur, io->k_comp, io->v_comp, io->kept_cnt,
                   io->out, ws, s);
}


// ---- comparison selectors -------------------------------------------------------
int32_t fkv_select_heuristic(const fkv_params_t* p, int32_t policy, uint64_t seed,
                             const int32_t* k_per_head, float* seg_score, int32_t* kept_idx,
                             int32_t* kept_cnt, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (policy != FKV_POLICY_UNIFORM && policy != FKV_POLICY_RANDOM) return FKV_ERR_INVALID_ARG;
  if (!d.token && d.static_token_mask) return FKV_ERR_UNSUPPORTED;
  if (!k_per_head || !kept_cnt || (!kept_idx && d.max_kept > 0) ||
      (policy == FKV_POLICY_RANDOM && !seg_score && d.nseg > 0))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return cuda_status(launch_heuristic(d, policy, seed, k_per_head, seg_score, kept_idx, kept_cnt,
                                      status_ptr(ws), static_cast<cudaStream_t>(stream)));
}

// ---- FP8 compressed cache ------------------------------------------------------
static bool fp8_supported(const Dims& d) {
  return d.bf16 && !d.token && !d.static_token_mask && d.D == 128;
}
static bool aligned4(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; }

int32_t fkv_compact_gather_fp8(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                               const int32_t* kept_idx, const int32_t* kept_cnt,
                               const fkv_fp8_cache_t* c, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!fp8_supported(d)) return FKV_ERR_UNSUPPORTED;
  if (!c || ((!k_hist || !v_hist) && d.N > 0) || (!kept_idx && d.max_kept > 0) || !kept_cnt)
    return FKV_ERR_INVALID_ARG;
  if (((!c->k_comp || !c->v_comp) && d.comp_rows > 0) ||
      ((!c->k_comp_scale || !c->v_comp_scale) && d.F > 0))
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(k_hist) || !aligned16(v_hist) || !aligned16(c->k_comp) ||
      !aligned16(c->v_comp) || !aligned4(c->k_comp_scale) || !aligned4(c->v_comp_scale))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  if (d.F == 0) return FKV_OK;  // nothing can be kept
  return cuda_status(launch_quant_kept(d, kept_idx, kept_cnt, k_hist, v_hist, *c, status_ptr(ws),
                                       static_cast<cudaStream_t>(stream)));
}

int32_t fkv_quantize_chunk_fp8(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                               const void* v_cur, const fkv_fp8_cache_t* c, void* ws,
                               void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!fp8_supported(d)) return FKV_ERR_UNSUPPORTED;
  if (!c || !q_cur || !k_cur || !v_cur || !c->q_cur || !c->q_scale || !c->k_cur || !c->v_cur ||
      !c->k_cur_scale || !c->v_cur_scale)
    return FKV_ERR_INVALID_ARG;
  if (!aligned16(q_cur) || !aligned16(k_cur) || !aligned16(v_cur) || !aligned16(c->q_cur) ||
      !aligned16(c->k_cur) || !aligned16(c->v_cur) || !aligned4(c->q_scale) ||
      !aligned4(c->k_cur_scale) || !aligned4(c->v_cur_scale))
    return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  return cuda_status(launch_quant_chunk(d, q_cur, k_cur, v_cur, *c, status_ptr(ws),
                                        static_cast<cudaStream_t>(stream)));
}

// Host-side checks of the e4m3 operands that the given steps use.
static int32_t check_fp8_cache(const Dims& d, const fkv_fp8_cache_t* c, bool comp, bool cur) {
  if (!c) return FKV_ERR_INVALID_ARG;
  if (comp) {
    if (((!c->k_comp || !c->v_comp) && d.comp_rows > 0) ||
        ((!c->k_comp_scale || !c->v_comp_scale) && d.F > 0))
      return FKV_ERR_INVALID_ARG;
    if (!aligned16(c->k_comp) || !aligned16(c->v_comp) || !aligned4(c->k_comp_scale) ||
        !aligned4(c->v_comp_scale))
      return FKV_ERR_INVALID_ARG;
  }
  if (cur) {
    if (!c->q_cur || !c->q_scale || !c->k_cur || !c->v_cur || !c->k_cur_scale || !c->v_cur_scale)
      return FKV_ERR_INVALID_ARG;
    if (!aligned16(c->q_cur) || !aligned16(c->k_cur) || !aligned16(c->v_cur) ||
        !aligned4(c->q_scale) || !aligned4(c->k_cur_scale) || !aligned4(c->v_cur_scale))
      return FKV_ERR_INVALID_ARG;
  }
  return FKV_OK;
}

int32_t fkv_attend_compressed_fp8(const fkv_params_t* p, const fkv_fp8_cache_t* c,
                                  const int32_t* kept_cnt, void* out, void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!fp8_supported(d) || d.T < 128) return FKV_ERR_UNSUPPORTED;
  if (!c || !kept_cnt || !out || !c->q_cur || !c->q_scale || !c->k_cur || !c->v_cur ||
      !c->k_cur_scale || !c->v_cur_scale)
    return FKV_ERR_INVALID_ARG;
  if (((!c->k_comp || !c->v_comp) && d.comp_rows > 0) ||
      ((!c->k_comp_scale || !c->v_comp_scale) && d.F > 0))
    return FKV_ERR_INVALID_ARG;
  const void* ptrs[] = {c->q_cur, c->k_cur, c->v_cur, c->k_comp, c->v_comp, out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FKV_ERR_INVALID_ARG;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  if (d.LH == 0 || d.Lq == 0) return FKV_OK;
  return cuda_status(launch_attend_fp8_sm100(d, *c, kept_cnt, out, status_ptr(ws),
                                             static_cast<cudaStream_t>(stream)));
}

int32_t fkv_step_fp8(const fkv_params_t* p, const fkv_step_io_t* io, const fkv_fp8_cache_t* c,
                     void* ws, void* stream) {
  Dims d;
  int32_t st = make_dims(p, &d);
  if (st != FKV_OK) return st;
  if (!fp8_supported(d) || d.T < 128) return FKV_ERR_UNSUPPORTED;
  if (!io) return FKV_ERR_INVALID_ARG;
  // every check before the first launch
  if (!io->q_cur || !io->k_cur || !io->v_cur || ((!io->k_hist || !io->v_hist) && d.N > 0) ||
      !io->k_per_head || (!io->seg_score && d.nseg > 0) || (!io->kept_idx && d.max_kept > 0) ||
      !io->kept_cnt || !io->out || !io->head_role || (!io->static_mask && d.F > 0))
    return FKV_ERR_INVALID_ARG;
  const void* ptrs[] = {io->q_cur, io->k_cur, io->v_cur, io->k_hist, io->v_hist, io->out};
  for (const void* ptr : ptrs)
    if (!aligned16(ptr)) return FKV_ERR_INVALID_ARG;
  if ((st = check_fp8_cache(d, c, true, true)) != FKV_OK) return st;
  if ((st = check_ws(d, ws)) != FKV_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = do_score(d, io->q_cur, io->q_score, io->k_hist, io->k_cur, io->head_role,
                     io->seg_score, ws, s)))
    return st;
  // as in fkv_step: every kernel after the first is a programmatic dependent
  Dims dp = d;
  dp.pdl = d.F > 0;
  if ((st = do_select(dp, io->seg_score, io->head_role, io->static_mask, io->k_per_head,
                      io->kept_idx, io->kept_cnt, ws, s)))
    return st;
  dp.pdl = true;
  // kept segments, the chunk's segments and its query rows: one launch
  if ((st = cuda_status(launch_quant_step(dp, io->kept_idx, io->kept_cnt, io->k_hist, io->v_hist,
                                          io->q_cur, io->k_cur, io->v_cur, *c, status_ptr(ws),
                                          s))))
    return st;
  return cuda_status(launch_attend_fp8_sm100(dp, *c, io->kept_cnt, io->out, status_ptr(ws), s));
}

}  // extern "C"
