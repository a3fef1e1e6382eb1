/*
 * fkv.h -- C ABI of the Forcing-KV chunk step for NVIDIA B200 (sm_100a).
 *
 * One call of fkv_step performs, for every (layer, head) of a chunk-
 * autoregressive video DiT, the hybrid head-wise KV-cache compression of
 * Forcing-KV and the chunk's attention over the compressed cache:
 *
 *   1. static heads keep a fixed, profiled set of history frames
 *      (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "关键模块" 2:
 *      structured static pruning, positions fixed once and extracted by mask);
 *   2. dynamic heads score every history frame ("segment") by the attention
 *      the current chunk's queries pay to it ("关键模块" 3: history grouped by
 *      frame, each group scored against the current queries);
 *   3. dynamic heads keep their top-k segments ("关键模块" 3: only the most
 *      similar few segments are kept);
 *   4. the kept K/V rows are compacted into a dense per-head cache
 *      ("输出与工程收益": the pruned KV replaces the original cache);
 *   5. the chunk's queries attend to that compressed cache followed by the
 *      chunk's own K/V ("输出与工程收益"; "与现有产品/工作流的接口" step 2).
 *
 * A token-granular variant (FKV_GRAN_TOKEN) implements Deep Forcing's
 * participative compression (bxzpzcl.cn/news/2125000, section 3.1): sink and
 * recent tokens kept whole, candidate tokens scored by phi_j = sum_r q_r.k_j
 * and the top C kept.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor argument is a DEVICE pointer owned by the caller.  The
 *    library never allocates, frees or synchronises the host (except
 *    fkv_read_status, which says so).  A buffer whose size is zero for the
 *    given params (e.g. k_comp when comp_rows == 0, seg_score when there is
 *    nothing to score) may be NULL.
 *  - Activations are contiguous row-major [L][H][rows][D]: bf16 (uint16
 *    storage) when dtype == FKV_DTYPE_BF16, float when FKV_DTYPE_FP32.  They
 *    must be 16-byte aligned.  L = num_layers, H = num_heads, D = head_dim.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    All work is enqueued asynchronously on it.
 *  - Return value: an fkv_status_t.  Host-side checks (null pointers, sizes,
 *    alignment, enums) run before anything is enqueued; on failure nothing is
 *    launched.  Checks that need device data (k out of range, kept rows above
 *    the capacity, segment ids out of range) cannot fail the call: the
 *    kernels clamp, record the first such error in the workspace status word,
 *    and the caller reads it with fkv_read_status.
 *  - Calls that run on the same workspace must not overlap on the GPU.
 */
#ifndef FKV_H_
#define FKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 3: adds fkv_fp8_cache_t and the three *_fp8 entry points;
 * 4: adds fkv_select_heuristic; 5: adds fkv_step_fp8;
 * 6: adds fkv_diag_attend_timeout, fkv_diag_mma_rate, fkv_diag_ex2_rate. */
#define FKV_ABI_VERSION 6

typedef enum fkv_status {
  FKV_OK = 0,
  FKV_ERR_INVALID_ARG = 1, /* null pointer, unknown enum, misaligned pointer  */
  FKV_ERR_SHAPE = 2,       /* sizes negative, inconsistent or above limits    */
  FKV_ERR_UNSUPPORTED = 3, /* valid request this build does not implement     */
  FKV_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed          */
  FKV_ERR_TIMEOUT = 5,     /* (device) a bounded wait gave up                 */
  FKV_ERR_WORKSPACE = 6,   /* workspace null, too small or not 256-B aligned  */
  FKV_ERR_DEVICE_ARG = 7   /* (device) k, segment id or capacity out of range */
} fkv_status_t;

typedef enum fkv_dtype { FKV_DTYPE_BF16 = 0, FKV_DTYPE_FP32 = 1 } fkv_dtype_t;

/* Segment = one latent frame of T tokens (Forcing-KV), or one token (the
 * participative variant, where every head is dynamic). */
typedef enum fkv_granularity { FKV_GRAN_FRAME = 0, FKV_GRAN_TOKEN = 1 } fkv_granularity_t;

/* fkv_params_t.flags bits. */
#define FKV_FLAG_SCORE_WITH_CHUNK 1 /* frame mode: the scoring softmax of each
                                       query row is normalised over the history
                                       keys AND the chunk's own keys (the
                                       attention the chunk computes); masses are
                                       still per history frame.  Default (0):
                                       history keys only. */
#define FKV_FLAG_STATIC_TOKEN_MASK 2 /* frame mode: static heads keep fixed TOKEN
                                       positions (e.g. chunk-boundary tokens):
                                       static_mask is [L][H][N], one byte per
                                       history token; every head's kept list
                                       then holds token ids (a dynamic head's
                                       kept frames expanded to their T tokens,
                                       ascending), kept_idx is [L][H][N],
                                       kept_cnt counts tokens, and the
                                       compressed cache, attention and
                                       fkv_cache_advance work on tokens
                                       (segment = 1 row).  seg_score stays
                                       [L][H][F]. */

typedef struct fkv_params {
  int32_t num_layers;    /* L >= 1: layers batched in one call (independent)  */
  int32_t num_heads;     /* H >= 1                                             */
  int32_t head_dim;      /* D: 128 for bf16; 4..128, multiple of 4, for fp32   */
  int32_t frame_tokens;  /* T >= 1: tokens per latent frame                    */
  int32_t hist_frames;   /* F >= 0: history frames; N = F*T history tokens     */
  int32_t chunk_frames;  /* Fc >= 1: chunk frames; Lq = Fc*T queries per head  */
  int32_t score_stride;  /* frame mode, >= 1: scoring queries are q_cur rows
                            0, s, 2s, ... (n_s = ceil(Lq / s) rows)            */
  int32_t n_score_q;     /* token mode, >= 1: rows of q_score per head         */
  int32_t sink_tokens;   /* token mode: S >= 0 first history tokens, kept      */
  int32_t recent_tokens; /* token mode: R >= 0 last history tokens, kept;
                            S + R <= N                                         */
  int32_t comp_rows;     /* rows per (layer, head) of k_comp / v_comp (>= 0)   */
  float scale;           /* softmax scale of the logits, finite and > 0, e.g.
                            1/sqrt(D)                                          */
  int32_t dtype;         /* fkv_dtype_t                                        */
  int32_t granularity;   /* fkv_granularity_t                                  */
  int32_t flags;         /* FKV_FLAG_* bits, 0 for the defaults                */
} fkv_params_t;

/* All inputs and outputs of fkv_step (device pointers, caller-owned). */
typedef struct fkv_step_io {
  const void* q_cur;          /* [L][H][Lq][D] chunk queries                    */
  const void* k_cur;          /* [L][H][Lq][D] chunk keys                       */
  const void* v_cur;          /* [L][H][Lq][D] chunk values                     */
  const void* k_hist;         /* [L][H][N][D] history keys, frame f = rows
                                 f*T .. f*T+T-1                                 */
  const void* v_hist;         /* [L][H][N][D] history values                    */
  const void* q_score;        /* token mode: [L][H][n_score_q][D]; else unused  */
  const uint8_t* head_role;   /* frame mode: [L][H], 0 = static, 1 = dynamic;
                                 unused (may be NULL) in token mode             */
  const uint8_t* static_mask; /* frame mode: [L][H][F], 1 = keep frame (read
                                 for static heads only); unused in token mode   */
  const int32_t* k_per_head;  /* [L][H]: frame mode: frames kept by a dynamic
                                 head (0..F); token mode: C (0..N-S-R)          */
  float* seg_score;           /* [L][H][nseg] segment scores (fkv_num_segments) */
  int32_t* kept_idx;          /* [L][H][max_kept] kept segment ids, ascending   */
  int32_t* kept_cnt;          /* [L][H] number of kept segments                 */
  void* k_comp;               /* [L][H][comp_rows][D] compressed keys           */
  void* v_comp;               /* [L][H][comp_rows][D] compressed values         */
  void* out;                  /* [L][H][Lq][D] attention output (q dtype)       */
} fkv_step_io_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* fkv_status_string(int32_t status);

/* FKV_ABI_VERSION of the loaded library. */
int32_t fkv_abi_version(void);

/* Validates params alone (no pointers) and returns the status fkv_step would
 * return for them. */
int32_t fkv_check_params(const fkv_params_t* p);

/* Scored segments per head: F (frame mode) or the candidate count N - S - R
 * (token mode).  Size of the last dimension of seg_score. */
int32_t fkv_num_segments(const fkv_params_t* p, int64_t* nseg);

/* Entries per head of kept_idx: F (frame mode) or N (token mode, where the
 * kept list holds token ids: sink, selected candidates, recent). */
int32_t fkv_max_kept(const fkv_params_t* p, int64_t* max_kept);

/* Compressed-cache rows per head needed for the worst case (every segment
 * kept): F*T in frame mode, N in token mode.  comp_rows may be smaller when
 * the caller knows its budgets; overflow is a device error (see above). */
int32_t fkv_max_comp_rows(const fkv_params_t* p, int64_t* rows);

/* Bytes of device workspace the entry points need for these params
 * (status word plus the scoring scratch).  Always >= 256. */
int32_t fkv_workspace_size(const fkv_params_t* p, size_t* bytes);

/* Number of kernel launches one fkv_step call enqueues for these params. */
int32_t fkv_step_launches(const fkv_params_t* p, int32_t* launches);

/* Diagnostic: y[i] = the FMA-pipe 2^x that the attention kernel uses for a
 * share of its softmax exponentials (Cody-Waite range reduction and a
 * degree-3 minimax polynomial; relative error <= 8.6e-5 for -126 <= x <= 127,
 * -inf -> +0), so that it can be tested against the hardware exp2.  x, y:
 * device arrays of n floats. */
int32_t fkv_exp2_emulated(const float* x, float* y, int64_t n, void* stream);

/* Diagnostic of the failure path: fkv_attend_compressed (bf16 tensor-core
 * kernel) with every bounded device wait limited to wait_cycles SM cycles
 * (10^4 .. 2*10^9; production calls use 2*10^9, about one second) and with
 * CTA 0 withholding the completion signal of its first logit tile, so that
 * the softmax's wait for it runs out.  The MMAs behind the signal are issued
 * and complete; nothing else is left outstanding.  Expected result: the call
 * returns FKV_OK, every CTA winds down (waiting, bounded, for its own copies
 * and MMAs, then freeing its tensor memory), and fkv_read_status reports
 * FKV_ERR_TIMEOUT with detail 0 (the CTA that gave up); `out` rows of the
 * work units CTA 0 owned are left unwritten, the other rows are the
 * attention.  No trap, no fault: the context stays usable.  fp32 params:
 * FKV_ERR_UNSUPPORTED. */
int32_t fkv_diag_attend_timeout(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                                const void* v_cur, const void* k_comp, const void* v_comp,
                                const int32_t* kept_cnt, void* out, int64_t wait_cycles, void* ws,
                                void* stream);

/* Diagnostics of the hardware rates the attention kernel's design rests on
 * (one CTA per SM; CTA 0 reports; no caller data is touched):
 *  - fkv_diag_mma_rate: one thread issues n_mma (8..4096, a multiple of 8)
 *    tcgen05.mma back to back into one fp32 accumulator in tensor memory.
 *    Shapes (bf16 unless noted): 0 = M128 N128 K16, A and B K-major in
 *    shared memory (the Q.K^T step); 1 = M128 N128 K16, A from tensor memory,
 *    B MN-major (the P.V step: V stored [keys][dims]); 2 = M128 N256; 3 =
 *    M128 N64; 4 = shape 0 with an MN-major B; 5 = shape 1 with a K-major B;
 *    6, 7 = shapes 0, 1 issued eight at a time through the attention
 *    kernel's own issue code; 8, 9 = the e4m3 attention's M128 N128 K32
 *    kind::f8f6f4 Q.K^T and P.V, four at a time through its issue code;
 *    10 = shape 0 with M = 64.
 *    busy != 0 keeps two more warps of the issuer's sub-partition running an
 *    FMA + ex2 loop meanwhile.  cycles: device int64[4]; cycles[0] = SM
 *    cycles to issue the n MMAs, cycles[1] = until they have completed.  ws:
 *    a workspace (>= 256 B, 256-B aligned) whose status word records
 *    FKV_ERR_TIMEOUT if the completion wait gave up.
 *  - fkv_diag_ex2_rate: `warps` (1..4) warps per SM sub-partition each run
 *    n (multiple of 8, <= 2^20) ex2.approx.ftz.f32 in 8 independent chains;
 *    cycles: device int64[2]; cycles[0] = SM cycles of one warp.
 * Sizes out of range: FKV_ERR_SHAPE. */
int32_t fkv_diag_mma_rate(int32_t shape, int32_t n_mma, int32_t busy, int64_t* cycles, void* ws,
                          void* stream);
int32_t fkv_diag_ex2_rate(int32_t n, int32_t warps, int64_t* cycles, void* stream);

/* Zeroes the workspace (status word included) on `stream`.  Call once after
 * allocating it; entry points never clear the status word themselves. */
int32_t fkv_workspace_init(void* ws, size_t bytes, void* stream);

/* Synchronises `stream`, then copies the workspace status word to the host:
 * *device_status = first device-side error recorded since the last init
 * (FKV_OK if none), *detail = the (layer*H + head) it was seen on, or -1.
 * Either output pointer may be NULL. */
int32_t fkv_read_status(const void* ws, void* stream, int32_t* device_status, int32_t* detail);

/* Step 2: segment scores.  Forcing-KV (ai-feeds.com/i/paper/2605.09681),
 * "关键模块" 3: a dynamic head's history is grouped by frame and each group
 * is scored by the current chunk's queries; Deep Forcing (bxzpzcl.cn/news/
 * 2125000) section 3.1 step 2 for the token variant's phi_j.
 * Frame mode (dynamic heads only; static rows of seg_score are written 0):
 *   seg_score[l][h][f] = sum_i sum_{j in frame f} softmax_j(scale * q_i . k_j),
 *   q_i = q_cur[l][h][i*score_stride], softmax over the N history keys (and
 *   the Lq rows of k_cur too with FKV_FLAG_SCORE_WITH_CHUNK; k_cur is unused
 *   and may be NULL otherwise).  q_score is unused (may be NULL).
 * Token mode (every head): seg_score[l][h][c] = sum_r q_score[l][h][r] .
 *   k_hist[l][h][S + c] for the candidates c = 0 .. N-S-R-1 (no scale).
 * Scores are float32.  Uses the scoring scratch of `ws`. */
int32_t fkv_score_segments(const fkv_params_t* p, const void* q_cur, const void* q_score,
                           const void* k_hist, const void* k_cur, const uint8_t* head_role,
                           float* seg_score, void* ws, void* stream);

/* fkv_score_segments without a workspace argument, for callers that cannot
 * allocate device memory (e.g. a plugin that a host runtime hands only its
 * input and output buffers, or a serving loop that has reserved all of HBM
 * up front).  The pages have no counterpart of this entry point: it is a
 * deployment convenience of this library.
 *
 * Same arguments, results and host-side checks as fkv_score_segments.  The
 * scratch lives in a static 16 MiB device array inside the library (held by
 * every GPU that loads the library until the process exits); sizes needing
 * more (fkv_workspace_size > 16 MiB, e.g. the 1080P layer or the 30-layer
 * 480P batch) are rejected with FKV_ERR_WORKSPACE and nothing is launched.  It calls no
 * cudaMalloc / cudaFree.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it for the
 *    life of the process; make that first call before any stream capture.
 *    The cached address belongs to the device's current CUDA context: after
 *    cudaDeviceReset (or anything else that destroys that context) it is
 *    stale, so do not call this entry point on a device after resetting it.
 *  - Every call on a device shares the one array and leaves its contents
 *    behind.  Each call first clears the 256-byte status block at the start
 *    of the array (a cudaMemsetAsync on `stream`); the partial statistics
 *    after it are written before they are read and need no clearing.  Calls
 *    that overlap on the GPU (different streams, or threads) race on the
 *    array and must be serialised by the caller.
 *  - There is no status word for the caller to read: a device-side failure
 *    of the scoring (a bounded wait that gave up) instead makes every dynamic
 *    head's scores NaN. */
int32_t fkv_score_segments_noalloc(const fkv_params_t* p, const void* q_cur, const void* q_score,
                                   const void* k_hist, const void* k_cur,
                                   const uint8_t* head_role, float* seg_score, void* stream);

/* Steps 1 and 3: kept segment lists.  Forcing-KV "关键模块" 2 (static heads:
 * fixed positions taken out by mask) and 3 (dynamic heads: the most similar
 * segments kept); Deep Forcing section 3.1 steps 1 and 3 (sink and recent
 * regions kept, top C = N - S - R candidates).
 * Frame mode: static heads keep the frames with static_mask == 1; dynamic
 *   heads keep the k_per_head[l][h] frames of largest seg_score, ties to the
 *   lower frame.  kept_idx[l][h][0..cnt) ascending, kept_cnt[l][h] = cnt.
 * Token mode: kept = [0, S) + (S + the C best candidates, ties to the lower
 *   index) + [N-R, N), ascending; kept_cnt = S + C + R.
 * Entries of kept_idx past kept_cnt are left untouched.
 * k out of range is clamped to [0, nseg] and recorded as FKV_ERR_DEVICE_ARG. */
int32_t fkv_select_topk(const fkv_params_t* p, const float* seg_score, const uint8_t* head_role,
                        const uint8_t* static_mask, const int32_t* k_per_head, int32_t* kept_idx,
                        int32_t* kept_cnt, void* ws, void* stream);

/* Step 4: compaction.  Forcing-KV "输出与工程收益": the pruned KV tensors
 * replace the original cache.  For each (l, h), copies the history rows of the kept
 * segments, in kept_idx order, into rows 0 .. kept_cnt*seg_len - 1 of
 * k_comp / v_comp (seg_len = T or 1).  Bit-exact copy.  Rows past that are
 * left untouched.  More rows than comp_rows: the copy is clamped and
 * FKV_ERR_DEVICE_ARG recorded. */
int32_t fkv_compact_gather(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                           const int32_t* kept_idx, const int32_t* kept_cnt, void* k_comp,
                           void* v_comp, void* ws, void* stream);

/* Step 5.  Forcing-KV "输出与工程收益" (the compressed KV takes the original
 * cache's place in the attention) and "与现有产品/工作流的接口" step 2.
 * out[l][h][i] = sum_j softmax_j(scale * q_i . key_j) value_j with the
 * keys = k_comp rows 0 .. kept_cnt*seg_len - 1 followed by the Lq rows of
 * k_cur (no causal mask), values likewise.  float32 accumulation; the output
 * is rounded to the activation dtype.  Compressed rows past the kept count
 * are never used. */
int32_t fkv_attend_compressed(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                              const void* v_cur, const void* k_comp, const void* v_comp,
                              const int32_t* kept_cnt, void* out, void* ws, void* stream);

/* Step 4 with temporal RoPE re-positioning of the kept keys (frame mode,
 * frame masks): the copy of fkv_compact_gather, except that the p-th of the
 * cnt kept frames of a head moves from frame kept_idx[p] to frame
 * F - cnt + p (the kept frames close up, ending right before the chunk), and
 * the temporal band of its keys -- the first n_pairs pairs of adjacent dims
 * (k[2i], k[2i+1]) taken as complex numbers -- is rotated by the angle
 * omega[i] * ((F - cnt + p) - kept_idx[p]); other dims and the values are
 * copied unchanged.  Deep Forcing (bxzpzcl.cn/news/2125000, section 2.2.2)
 * rotates cached keys' time component by the phase exp(i omega_t delta) when
 * their temporal offset changes (section 3.2 item 3: also for selected
 * tokens).  omega: device float[n_pairs], the model's temporal RoPE
 * frequencies; 0 <= 2*n_pairs <= D.  Rotation in fp32, rounded once to the
 * activation dtype.  Token mode / token masks: FKV_ERR_UNSUPPORTED. */
int32_t fkv_compact_gather_rope(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                                const int32_t* kept_idx, const int32_t* kept_cnt,
                                const float* omega, int32_t n_pairs, void* k_comp, void* v_comp,
                                void* ws, void* stream);

/* Cache lifecycle: the history cache for the next chunk.  For each (l, h),
 * k_next[l][h] = the last (out_segments - chunk_segs) kept segments of the
 * compressed cache (rows of k_comp, in order), followed by the Lq rows of the
 * chunk's own k_cur; the same for v.  chunk_segs = Fc (frame mode) or Lq
 * (token mode); out_segments counts segments of the result, so the next
 * call's history is out_segments frames (frame mode: hist_frames =
 * out_segments) or tokens, the older kept segments being dropped (a fixed
 * window).  The compressed KV replaces the cache (Forcing-KV,
 * "输出与工程收益") and the new chunk joins it; the window follows Deep
 * Forcing's budget of 70-80% of a sliding window (section 5.1).
 * k_next, v_next: [L][H][out_segments*seg_len][D]; they must not overlap the
 * inputs.  A head that kept fewer than out_segments - chunk_segs segments gets
 * zero rows there and FKV_ERR_DEVICE_ARG is recorded.  k_comp / v_comp may
 * be NULL when out_segments == chunk_segs (chunk only); kept_cnt is always
 * required.
 * Denoising steps after the first reuse a chunk's selection and compressed
 * cache by calling fkv_attend_compressed alone. */
int32_t fkv_cache_advance(const fkv_params_t* p, const void* k_comp, const void* v_comp,
                          const int32_t* kept_cnt, const void* k_cur, const void* v_cur,
                          int64_t out_segments, void* k_next, void* v_next, void* ws,
                          void* stream);

/* Steps 1-5 in one call (Forcing-KV "方法": "输入与整体流程", "关键模块" 2-3,
 * "输出与工程收益"): score (dynamic / token heads), select, compact, attend,
 * all enqueued on `stream`, each step after the one it reads from. */
int32_t fkv_step(const fkv_params_t* p, const fkv_step_io_t* io, void* ws, void* stream);

/* ---- Comparison selectors --------------------------------------------------
 * Forcing-KV (ai-feeds.com/i/paper/2605.09681, "与基线对比及工程启示", first
 * item) measures itself against uniform eviction and random dropping at the
 * same compression ratio; the pages define neither.  Reading: every head keeps
 * its budget k_per_head[l][h] (k frames in frame mode, C candidate tokens in
 * token mode) whatever its role, and the output has the format of
 * fkv_select_topk (kept_idx ascending, entries past kept_cnt untouched; token
 * mode adds the sink [0, S) and recent [N-R, N) tokens).
 *   FKV_POLICY_UNIFORM: of the n segments (frames, or candidates) keep
 *     floor(i * n / k) for i < k; seg_score is not used (may be NULL).
 *   FKV_POLICY_RANDOM: keep the k segments of largest priority, ties to the
 *     lower index, where the priority of segment s of head lh is the first
 *     64-bit word w of Philox4x64-10 (Salmon et al., "Parallel random
 *     numbers: as easy as 1, 2, 3", SC 2011) at counter (s, lh, 0, 0) and
 *     key (seed, 0), as (w >> 40) * 2^-24.  The priorities are written to
 *     seg_score (float [L*H][nseg], device) and then ranked.
 * Frame mode with FKV_FLAG_STATIC_TOKEN_MASK: FKV_ERR_UNSUPPORTED.  An unknown
 * policy: FKV_ERR_INVALID_ARG.  k out of range: clamped, FKV_ERR_DEVICE_ARG. */
typedef enum fkv_policy {
  FKV_POLICY_UNIFORM = 0,
  FKV_POLICY_RANDOM = 1
} fkv_policy_t;

int32_t fkv_select_heuristic(const fkv_params_t* p, int32_t policy, uint64_t seed,
                             const int32_t* k_per_head, float* seg_score, int32_t* kept_idx,
                             int32_t* kept_cnt, void* ws, void* stream);

/* ---- FP8 (e4m3) compressed cache ------------------------------------------
 * Forcing-KV (ai-feeds.com/i/paper/2605.09681), "与现有产品/工作流的接口" item
 * 3: the compression composes with KV quantization; the pages fix no format.
 * Reading: OCP FP8 E4M3 (largest finite 448), round to nearest even,
 * saturating; one fp32 scale per (l, h, segment) for K and one for V, where a
 * segment is a kept history frame or a frame of the current chunk, and one per
 * query row for Q.  Scale s = amax / 448 over the block (1 for an all-zero
 * block); code = e4m3(x * (448 / amax)), each division and the product one
 * correctly rounded fp32 operation.  The value a code stands for is
 * e4m3(code) * s.
 *
 * Operands of the fp8 attention, all device memory owned by the caller, all
 * code arrays row-major with D = 128 bytes per row and 16-byte aligned:
 *   k_comp, v_comp  uint8 [L*H][comp_rows][D]  kept history rows, segment p
 *                   (the p-th kept frame) in rows [p*T, (p+1)*T)
 *   k_comp_scale, v_comp_scale  float [L*H][F]  scale of kept segment p
 *   k_cur, v_cur    uint8 [L*H][Lq][D]         the chunk's own rows
 *   k_cur_scale, v_cur_scale    float [L*H][Fc] scale of chunk frame g
 *   q_cur           uint8 [L*H][Lq][D]         the chunk's queries
 *   q_scale         float [L*H][Lq]            scale of query row r
 * Supported: bf16 activations, head_dim 128, frame granularity with frame
 * masks; otherwise FKV_ERR_UNSUPPORTED.  The attention also needs
 * frame_tokens >= 128 (a 128-key block spans at most two segments). */
typedef struct fkv_fp8_cache {
  void* k_comp;
  void* v_comp;
  float* k_comp_scale;
  float* v_comp_scale;
  void* k_cur;
  void* v_cur;
  float* k_cur_scale;
  float* v_cur_scale;
  void* q_cur;
  float* q_scale;
} fkv_fp8_cache_t;

/* Step 4 into the fp8 cache: for each (l, h) and p < kept_cnt[l][h], the
 * frame kept_idx[l][h][p] of k_hist / v_hist (bf16 [L*H][F*T][D]) is
 * quantized as one segment into rows [p*T, (p+1)*T) of c->k_comp / c->v_comp
 * and its scales into c->k_comp_scale[l][h][p] / c->v_comp_scale[l][h][p].
 * Rows and scales of segments p >= kept_cnt are not written.  A kept_cnt or
 * kept_idx entry out of range is reported as FKV_ERR_DEVICE_ARG through the
 * workspace status and that segment skipped.  c: host struct, only the
 * k_comp / v_comp / *_comp_scale members are used. */
int32_t fkv_compact_gather_fp8(const fkv_params_t* p, const void* k_hist, const void* v_hist,
                               const int32_t* kept_idx, const int32_t* kept_cnt,
                               const fkv_fp8_cache_t* c, void* ws, void* stream);

/* The chunk's own operands in fp8: k_cur / v_cur (bf16 [L*H][Lq][D]) frame by
 * frame into c->k_cur / c->v_cur with per-frame scales, q_cur (bf16
 * [L*H][Lq][D]) row by row into c->q_cur / c->q_scale.  c: host struct, only
 * the *_cur members and q_scale are used. */
int32_t fkv_quantize_chunk_fp8(const fkv_params_t* p, const void* q_cur, const void* k_cur,
                               const void* v_cur, const fkv_fp8_cache_t* c, void* ws,
                               void* stream);

/* Step 5 over the fp8 cache: out (bf16 [L*H][Lq][D]) = softmax attention of
 * the dequantised queries over the dequantised keys = kept rows
 * [0, kept_cnt*T) of k_comp then the Lq rows of k_cur, with values likewise,
 * scale p->scale.  Tensor cores (kind::f8f6f4) with fp32 accumulation; the
 * probabilities are rounded to e4m3 before the P.V product (after a per-head
 * rescale by v_scale / max v_scale), so the result differs from the exact
 * attention over the dequantised cache by that rounding. */
int32_t fkv_attend_compressed_fp8(const fkv_params_t* p, const fkv_fp8_cache_t* c,
                                  const int32_t* kept_cnt, void* out, void* ws, void* stream);

/* Steps 1-5 with the e4m3 cache in one call: score and select as fkv_step,
 * then the work of fkv_compact_gather_fp8 and fkv_quantize_chunk_fp8 (one
 * launch) and fkv_attend_compressed_fp8, all enqueued on `stream` in that
 * order, each kernel after the first a programmatic dependent of the one
 * before (as in fkv_step).  io as
 * for fkv_step (frame mode), except that io->k_comp / io->v_comp are not used
 * (may be NULL); c holds every e4m3 operand.  Same support limits as
 * fkv_attend_compressed_fp8; every host-side check runs before the first
 * launch. */
int32_t fkv_step_fp8(const fkv_params_t* p, const fkv_step_io_t* io, const fkv_fp8_cache_t* c,
                     void* ws, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* FKV_H_ */
