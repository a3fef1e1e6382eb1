"""Plain float64 oracle of one Forcing-KV chunk step (test infrastructure).

Every function works on one (layer, head) at a time with numpy float64 and is
written as the definition it follows, with no blocking beyond splitting
independent query rows, no fusion and no reordering of the sums the
definitions state.  Inputs are the exact float64 upcast of what the CUDA path
reads (bf16 or fp32), so the only differences between the two sides come from
the CUDA path's own rounding.

Readings of points the pages leave open (each listed in the design notes):
  * segment score = softmax attention mass over the HISTORY keys only,
    summed over the scoring queries and over the tokens of the frame;
  * scoring queries = rows 0, s, 2s, ... of the current chunk's queries;
  * top-k, ties to the lower segment index, kept list ascending;
  * the compressed cache holds the kept segments in ascending order;
  * the chunk's queries attend, without a causal mask, to the compressed
    history followed by the chunk's own keys;
  * token variant: phi_j = sum_r q_r . k_j with no scale and no softmax, sink
    and recent tokens always kept.
"""
from __future__ import annotations

from typing import Dict, List, Optional

import numpy as np

# Query rows per block when a score matrix is materialised (rows are
# independent, so splitting them changes no arithmetic).
_ROW_BLOCK = 512


def static_keep(mask_row: np.ndarray) -> np.ndarray:
    """Kept frames of a static head: ascending f with mask[f] == 1.

    Forcing-KV, "关键模块" 2 (static structural pruning): the kept positions
    are fixed once by profiling and taken out by mask at inference.
    """
    return np.flatnonzero(np.asarray(mask_row) != 0).astype(np.int64)


def frames_to_tokens(frames: np.ndarray, T: int) -> np.ndarray:
    """Token ids of the given frames, in order (frame f = tokens f*T .. f*T+T-1)."""
    if len(frames) == 0:
        return np.zeros(0, dtype=np.int64)
    return (np.asarray(frames)[:, None] * T + np.arange(T)[None, :]).reshape(-1).astype(np.int64)


def scoring_queries(q_cur: np.ndarray, stride: int) -> np.ndarray:
    """Rows 0, stride, 2*stride, ... of the chunk's queries (the scoring set)."""
    return q_cur[0::stride]


def segment_mass(q_rows: np.ndarray, k_hist: np.ndarray, T: int, scale: float,
                 k_chunk: Optional[np.ndarray] = None) -> np.ndarray:
    """Per-frame softmax attention mass of a dynamic head.

    Forcing-KV, "关键模块" 3 (dynamic similarity pruning): the history cache is
    grouped by frame and each group gets the attention score of the current
    queries.  Read as: z_ij = scale * q_i . k_j over all N history keys,
    p_ij = exp(z_ij) / sum_j' exp(z_ij') (per query row, history keys only),
    mass_f = sum_i sum_{j in frame f} p_ij.
    With k_chunk given, the normaliser of each row also runs over the chunk's
    own keys (the attention the chunk actually computes); the masses are still
    those of the history frames.

    q_rows [n_s][D], k_hist [F*T][D], k_chunk [Lq][D] or None -> mass [F].
    """
    n_s = q_rows.shape[0]
    N = k_hist.shape[0]
    F = N // T
    if F == 0:  # empty history: nothing to score
        return np.zeros(0)
    keys = k_hist if k_chunk is None else np.concatenate([k_hist, k_chunk], axis=0)
    per_row = np.empty((n_s, F), dtype=np.float64)
    for r0 in range(0, n_s, _ROW_BLOCK):
        z = scale * (q_rows[r0:r0 + _ROW_BLOCK] @ keys.T)
        z = z - z.max(axis=1, keepdims=True)
        e = np.exp(z)
        p = e / e.sum(axis=1, keepdims=True)
        per_row[r0:r0 + _ROW_BLOCK] = p[:, :N].reshape(p.shape[0], F, T).sum(axis=2)
    return per_row.sum(axis=0)


def top_k(scores: np.ndarray, k: int) -> np.ndarray:
    """The k best segments, ties to the lower index, returned ascending.

    Forcing-KV, "关键模块" 3: only the highest-scoring few segments are kept.
    Order by (-score, index) -- a stable sort of -score -- take k, re-sort.
    """
    order = np.argsort(-np.asarray(scores, dtype=np.float64), kind="stable")
    return np.sort(order[:k]).astype(np.int64)


def participative_phi(q_score: np.ndarray, k_cand: np.ndarray) -> np.ndarray:
    """phi_j = sum_r q_r^T k_j over the scoring queries r (no scale, no softmax).

    Deep Forcing, section 3.1 step 2 (importance score of a candidate token).
    q_score [R][D], k_cand [n][D] -> phi [n].
    """
    phi = np.zeros(k_cand.shape[0], dtype=np.float64)
    for r0 in range(0, q_score.shape[0], _ROW_BLOCK):
        phi += (q_score[r0:r0 + _ROW_BLOCK] @ k_cand.T).sum(axis=0)
    return phi


def token_keep(phi_cand: np.ndarray, N: int, sink: int, recent: int, C: int) -> np.ndarray:
    """Kept token indices: sink [0, S), the top-C candidates, recent [N-R, N).

    Deep Forcing, section 3.1 steps 1 and 3: sink and recent regions are kept
    whole, the candidate region keeps its C best tokens (C = N - S - R with N
    the budget).  Candidate i is history token sink + i.  Ascending output.
    """
    chosen = sink + top_k(phi_cand, C)
    return np.concatenate([np.arange(sink), chosen, np.arange(N - recent, N)]).astype(np.int64)


def compact(kv_hist: np.ndarray, kept: np.ndarray, seg_len: int) -> np.ndarray:
    """The compressed cache: the kept segments' rows, concatenated in order.

    Forcing-KV, "输出与工程收益": the pruned KV replaces the original cache.
    kv_hist [N][D], kept [cnt] segment ids, seg_len rows per segment.
    """
    if len(kept) == 0:
        return kv_hist[:0].copy()
    return np.concatenate([kv_hist[s * seg_len:(s + 1) * seg_len] for s in kept], axis=0)


def rope_shift(keys: np.ndarray, omega: np.ndarray, delta: float) -> np.ndarray:
    """Temporal RoPE re-positioning of keys by delta frames.

    Deep Forcing (bxzpzcl.cn/news/2125000), section 2.2.2 (and 3.2 item 3 for
    selected tokens): the time component of a cached key is multiplied by the
    phase exp(i * omega_t * delta).  Read as: the first len(omega) pairs of
    adjacent dims (k[2i], k[2i+1]) are complex numbers k[2i] + i k[2i+1], each
    rotated by the angle omega[i] * delta; the other dims are unchanged.
    keys [rows][D] -> [rows][D].
    """
    out = np.array(keys, dtype=np.float64, copy=True)
    n = len(omega)
    ang = np.asarray(omega, dtype=np.float64) * float(delta)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = out[:, 0:2 * n:2].copy(), out[:, 1:2 * n:2].copy()
    out[:, 0:2 * n:2] = x0 * c - x1 * s
    out[:, 1:2 * n:2] = x0 * s + x1 * c
    return out


def compact_repositioned(k_hist: np.ndarray, kept: np.ndarray, T: int, F: int,
                         omega: np.ndarray) -> np.ndarray:
    """Compressed keys with their temporal position re-assigned: the p-th of
    cnt kept frames moves from frame kept[p] to frame F - cnt + p (the kept
    frames close up, ending right before the chunk at frame F), and its keys
    are rotated by rope_shift with delta = (F - cnt + p) - kept[p]."""
    cnt = len(kept)
    parts = [rope_shift(k_hist[f * T:(f + 1) * T], omega, (F - cnt + p) - f)
             for p, f in enumerate(kept)]
    if not parts:
        return k_hist[:0].copy()
    return np.concatenate(parts, axis=0)


def attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float) -> np.ndarray:
    """o_i = sum_j softmax_j(scale * q_i . k_j) v_j, max-subtracted, float64.

    Forcing-KV, "输出与工程收益" and the integration step of "与现有产品/工作流
    的接口": attention of the chunk over the compressed cache.
    """
    out = np.empty((q.shape[0], values.shape[1]), dtype=np.float64)
    for r0 in range(0, q.shape[0], _ROW_BLOCK):
        z = scale * (q[r0:r0 + _ROW_BLOCK] @ keys.T)
        z = z - z.max(axis=1, keepdims=True)
        e = np.exp(z)
        out[r0:r0 + _ROW_BLOCK] = (e @ values) / e.sum(axis=1, keepdims=True)
    return out


def advance(comp: np.ndarray, kept_count: int, seg_len: int, chunk: np.ndarray,
            out_segments: int) -> np.ndarray:
    """The next history cache of one head: the most recent kept segments of the
    compressed cache followed by the chunk's own keys (or values).

    Forcing-KV, "输出与工程收益": the compressed KV replaces the original cache;
    the chunk just generated joins the history for the next chunk
    ("输入与整体流程": history KV grows frame by frame); a window keeps the
    cache bounded (Deep Forcing, section 5.1: a budget of 70-80% of the
    sliding window).  out_segments counts segments (frames, or tokens) of the
    result, chunk segments included; the oldest kept segments are dropped.
    comp [>= kept_count*seg_len][D], chunk [chunk_rows][D].
    """
    chunk_segs = chunk.shape[0] // seg_len
    keep = out_segments - chunk_segs
    assert 0 <= keep <= kept_count
    old = comp[(kept_count - keep) * seg_len:kept_count * seg_len]
    return np.concatenate([old, chunk], axis=0)


def head_keep(*, granularity: str, dynamic: bool, mask_row, k: int, q_cur, k_hist,
              T: int, scale: float, score_stride: int = 1, q_score=None,
              sink: int = 0, recent: int = 0, k_chunk=None, token_static_mask: bool = False):
    """Selection for one (layer, head): (kept segment ids, segment scores or None).
    k_chunk: include the chunk's own keys in the scoring normaliser.
    token_static_mask: static heads keep the tokens of a per-token mask (fixed
    positions such as chunk-boundary tokens, Forcing-KV "关键模块" 1-2) and
    every head's kept list is in tokens (a dynamic head's kept frames
    expanded to their tokens)."""
    N = k_hist.shape[0]
    if granularity == "frame" and token_static_mask:
        if not dynamic:
            return static_keep(mask_row), None
        mass = segment_mass(scoring_queries(q_cur, score_stride), k_hist, T, scale, k_chunk)
        return frames_to_tokens(top_k(mass, k), T), mass
    if granularity == "frame":
        if not dynamic:
            return static_keep(mask_row), None
        mass = segment_mass(scoring_queries(q_cur, score_stride), k_hist, T, scale, k_chunk)
        return top_k(mass, k), mass
    phi = participative_phi(q_score, k_hist[sink:N - recent])
    return token_keep(phi, N, sink, recent, k), phi


def step(q_cur, k_cur, v_cur, k_hist, v_hist, head_role, static_mask, k_per_head, *,
         T: int, granularity: str, scale: float, score_stride: int = 1,
         q_score=None, sink: int = 0, recent: int = 0,
         rows: Optional[np.ndarray] = None, heads=None) -> Dict[str, object]:
    """The whole chunk step for [L][H] heads.

    Arrays are float64 [L][H][rows][D]; head_role [L][H] (1 = dynamic),
    static_mask [L][H][F], k_per_head [L][H].  ``rows`` restricts the attention
    output to those query rows (sampled checks of large workloads); ``heads``
    restricts the work to a list of (l, h).

    Returns a dict: ``kept`` {(l,h): ascending segment ids}, ``score``
    {(l,h): segment scores (dynamic / token heads)}, ``out`` {(l,h): [rows][D]}.
    """
    L, H = head_role.shape
    seg_len = T if granularity == "frame" else 1
    kept: Dict[tuple, np.ndarray] = {}
    score: Dict[tuple, np.ndarray] = {}
    out: Dict[tuple, np.ndarray] = {}
    todo = heads if heads is not None else [(l, h) for l in range(L) for h in range(H)]
    for (l, h) in todo:
        ks, sc = head_keep(
            granularity=granularity, dynamic=bool(head_role[l, h]),
            mask_row=static_mask[l, h], k=int(k_per_head[l, h]), q_cur=q_cur[l, h],
            k_hist=k_hist[l, h], T=T, scale=scale, score_stride=score_stride,
            q_score=None if q_score is None else q_score[l, h], sink=sink, recent=recent)
        kept[(l, h)] = ks
        if sc is not None:
            score[(l, h)] = sc
        keys = np.concatenate([compact(k_hist[l, h], ks, seg_len), k_cur[l, h]], axis=0)
        vals = np.concatenate([compact(v_hist[l, h], ks, seg_len), v_cur[l, h]], axis=0)
        q = q_cur[l, h] if rows is None else q_cur[l, h][rows]
        out[(l, h)] = attention(q, keys, vals, scale)
    return {"kept": kept, "score": score, "out": out}


def kept_rows(kept: np.ndarray, granularity: str, T: int) -> int:
    """Rows of the compressed cache of one head."""
    return len(kept) * (T if granularity == "frame" else 1)


__all__: List[str] = [
    "static_keep", "scoring_queries", "segment_mass", "top_k", "participative_phi",
    "token_keep", "compact", "attention", "advance", "head_keep", "step", "kept_rows",
    "frames_to_tokens", "rope_shift", "compact_repositioned",
]
