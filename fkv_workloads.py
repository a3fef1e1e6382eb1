"""Seeded synthetic inputs for one Forcing-KV chunk step.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no scoring, no selection, no gather, no attention), so both
sides of every parity check -- the fp64 CPU oracle and the CUDA library -- can be
fed from it without sharing any computation.

Shapes stand in for the workloads named on the pages: a Wan-1.3B-style
Self-Forcing DiT at 480P (30x52 latent grid = 1560 tokens per latent frame) and
1080P (68x120 = 8160 tokens per frame), a chunk of 3 latent frames and an
18-frame history cache (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
"输入与整体流程"), and a 40-head 14B-shaped model for the token-level
participative variant (Deep Forcing, bxzpzcl.cn/news/2125000, section 3.1).
The pages measure with trained models and VBench; neither is used here, the
synthetic tensors below replace them.

Value recipe (all draws from ``numpy.random.default_rng(seed)`` (PCG64) in the
order listed, generated as float32 and rounded once, round-to-nearest-even, to
bfloat16 by torch for the bf16 workloads):

* video-style workloads (480P, 30-layer, 1080P, token 14B), per layer:
    1. head roles: ``perm = rng.permutation(H)``; ``perm[:n_static]`` are static
       (frame workloads only; the token workload has no static heads),
    2. Q_cur ~ N(0, 1), shape [H][Fc*T][D],
    3. for K then V: per-(head, frame) mean mu ~ N(0, 0.5^2) [H][F+Fc][D],
       innovations eta ~ N(0, 1) [H][F+Fc][D], token noise z ~ N(0, 1)
       [H][(F+Fc)*T][D]; drift d_0 = 0, d_f = 0.7 d_{f-1} + 0.3 eta_f;
       value[h, f*T + t] = mu[h, f] + d[h, f] + z[h, f*T + t].  Frames 0..F-1
       form the history cache, frames F..F+Fc-1 the current chunk,
    4. token workload only: q_score ~ N(0, 1), shape [H][n_score_q][D].
* tiny fp32 workload: Q_cur, K_hist, V_hist, K_cur, V_cur ~ N(0, 1) in that
  order, then a per-(head, frame) mean ~ N(0, 0.5^2) added to the history K.
"""
from __future__ import annotations

import concurrent.futures as _cf
import dataclasses
import os
from typing import Dict, Optional, Sequence, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes and selection budgets of one chunk step.

    L layers, H heads, D head dim, T tokens per latent frame, F history frames,
    Fc frames in the current chunk.  ``granularity`` is "frame" (Forcing-KV:
    a segment is one latent frame of T tokens) or "token" (participative
    variant: a segment is one token).
    """

    name: str
    L: int
    H: int
    D: int
    T: int
    F: int
    Fc: int
    dtype: str  # "bf16" or "fp32"
    granularity: str  # "frame" or "token"
    seed: int
    layer_seeds: Optional[Tuple[int, ...]] = None
    n_static: int = 0
    fixed_static_heads: Optional[Tuple[int, ...]] = None
    static_frames: Tuple[int, ...] = ()
    k_dynamic: int = 0
    score_stride: int = 1
    n_score_q: int = 0
    sink_tokens: int = 0
    recent_tokens: int = 0
    keep_tokens: int = 0  # C in the participative variant
    style: str = "video"  # "video" or "tiny"
    score_with_chunk: bool = False  # chunk keys in the scoring normaliser
    # static heads keep tokens: every token of frame 0 and the first and last
    # T/8 tokens of each other history frame (a chunk-boundary-like pattern)
    static_token_mask: bool = False

    @property
    def N(self) -> int:
        """History tokens per head."""
        return self.F * self.T

    @property
    def Lq(self) -> int:
        """Queries (and own keys) of the current chunk per head."""
        return self.Fc * self.T

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    @property
    def n_segments(self) -> int:
        """Scored segments per head: frames, or candidate tokens."""
        if self.granularity == "frame":
            return self.F
        return self.N - self.sink_tokens - self.recent_tokens

    def seeds(self) -> Tuple[int, ...]:
        if self.layer_seeds is not None:
            return self.layer_seeds
        return tuple(self.seed + l for l in range(self.L))


# Static keep pattern of the 480P/1080P workloads: frame 0 as a sink, then the
# first and last frame of each 3-frame history chunk 1-3, 4-6, ..., 13-15, and
# the 2-frame tail 16-17, i.e. 13 of 18 frames.
STATIC_FRAMES_18 = (0, 1, 3, 4, 6, 7, 9, 10, 12, 13, 15, 16, 17)

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload(
        name="tiny", L=1, H=4, D=64, T=32, F=6, Fc=1, dtype="fp32",
        granularity="frame", seed=0, fixed_static_heads=(0, 1),
        static_frames=(0, 5), k_dynamic=2, score_stride=1, style="tiny"),
    "480p": Workload(
        name="480p", L=1, H=12, D=128, T=1560, F=18, Fc=3, dtype="bf16",
        granularity="frame", seed=1, n_static=6, static_frames=STATIC_FRAMES_18,
        k_dynamic=13, score_stride=16),
    "480p_30layer": Workload(
        name="480p_30layer", L=30, H=12, D=128, T=1560, F=18, Fc=3, dtype="bf16",
        granularity="frame", seed=1000, n_static=6, static_frames=STATIC_FRAMES_18,
        k_dynamic=13, score_stride=16),
    "1080p": Workload(
        name="1080p", L=1, H=12, D=128, T=8160, F=18, Fc=3, dtype="bf16",
        granularity="frame", seed=2, n_static=6, static_frames=STATIC_FRAMES_18,
        k_dynamic=13, score_stride=32),
    "token14b": Workload(
        name="token14b", L=1, H=40, D=128, T=1560, F=18, Fc=3, dtype="bf16",
        granularity="token", seed=3, n_score_q=1560, sink_tokens=3 * 1560,
        recent_tokens=3 * 1560,
        # budget N = 75% of the 21-frame window, C = N - S - R
        keep_tokens=(3 * 21 * 1560) // 4 - 2 * 3 * 1560),
}


# Options of the 480P workload (same inputs, other readings of the method).
WORKLOADS["480p_chunknorm"] = dataclasses.replace(WORKLOADS["480p"], name="480p_chunknorm",
                                                  score_with_chunk=True)
WORKLOADS["480p_tokenmask"] = dataclasses.replace(WORKLOADS["480p"], name="480p_tokenmask",
                                                  static_token_mask=True)


def get(name: str) -> Workload:
    return WORKLOADS[name]


def scaled(w: Workload, **changes) -> Workload:
    """The same recipe with some sizes changed (edge and small parity cases)."""
    return dataclasses.replace(w, **changes)


def _torch_dtype(w: Workload):
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def _video_kv(rng, H, frames, T, D):
    mu = 0.5 * rng.standard_normal((H, frames, D), dtype=np.float32)
    eta = rng.standard_normal((H, frames, D), dtype=np.float32)
    z = rng.standard_normal((H, frames * T, D), dtype=np.float32)
    drift = np.zeros((H, frames, D), dtype=np.float32)
    for f in range(1, frames):
        drift[:, f] = 0.7 * drift[:, f - 1] + 0.3 * eta[:, f]
    z = z.reshape(H, frames, T, D)
    z += (mu + drift)[:, :, None, :]
    return z.reshape(H, frames * T, D)


def _layer(w: Workload, seed: int):
    """Draws one layer.  Returns float32 numpy arrays and the role / mask rows."""
    rng = np.random.default_rng(seed)
    H, D, T, F, Fc = w.H, w.D, w.T, w.F, w.Fc
    role = np.ones(H, dtype=np.uint8)  # 1 = dynamic, 0 = static
    if w.granularity == "frame":
        if w.fixed_static_heads is not None:
            role[list(w.fixed_static_heads)] = 0
        else:
            perm = rng.permutation(H)
            role[perm[: w.n_static]] = 0
    out = {}
    if w.style == "tiny":
        out["q_cur"] = rng.standard_normal((H, Fc * T, D), dtype=np.float32)
        k_hist = rng.standard_normal((H, F * T, D), dtype=np.float32)
        out["v_hist"] = rng.standard_normal((H, F * T, D), dtype=np.float32)
        out["k_cur"] = rng.standard_normal((H, Fc * T, D), dtype=np.float32)
        out["v_cur"] = rng.standard_normal((H, Fc * T, D), dtype=np.float32)
        mu = 0.5 * rng.standard_normal((H, F, D), dtype=np.float32)
        k_hist = (k_hist.reshape(H, F, T, D) + mu[:, :, None, :]).reshape(H, F * T, D)
        out["k_hist"] = k_hist
    else:
        out["q_cur"] = rng.standard_normal((H, Fc * T, D), dtype=np.float32)
        k_all = _video_kv(rng, H, F + Fc, T, D)
        v_all = _video_kv(rng, H, F + Fc, T, D)
        out["k_hist"], out["k_cur"] = k_all[:, : F * T], k_all[:, F * T:]
        out["v_hist"], out["v_cur"] = v_all[:, : F * T], v_all[:, F * T:]
        if w.granularity == "token":
            out["q_score"] = rng.standard_normal((H, w.n_score_q, D), dtype=np.float32)
    mask = np.zeros((H, F * T if w.static_token_mask else F), dtype=np.uint8)
    kph = np.zeros(H, dtype=np.int32)
    if w.granularity == "frame":
        edge = max(1, T // 8)
        for h in range(H):
            if role[h] == 0:
                if w.static_token_mask:
                    tok = mask[h].reshape(F, T)
                    tok[:, :edge] = 1
                    tok[:, T - edge:] = 1
                    if F > 0:
                        tok[0] = 1
                else:
                    mask[h, list(w.static_frames)] = 1
            else:
                kph[h] = w.k_dynamic
    else:
        kph[:] = w.keep_tokens
    return out, role, mask, kph


def generate(w: Workload, threads: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """All inputs of one chunk step as contiguous CPU tensors.

    Activations are [L][H][rows][D] in the workload's dtype (bf16 values are the
    RNE rounding of the float32 draws).  ``head_role`` is uint8 [L][H]
    (1 = dynamic), ``static_mask`` uint8 [L][H][F], ``k_per_head`` int32 [L][H]
    (segments kept per dynamic head: k frames, or C tokens).
    Layers are drawn in parallel threads, each from its own seed, so the result
    does not depend on ``threads``.
    """
    dt = _torch_dtype(w)
    L, H, D = w.L, w.H, w.D
    shapes = {
        "q_cur": (L, H, w.Lq, D), "k_cur": (L, H, w.Lq, D), "v_cur": (L, H, w.Lq, D),
        "k_hist": (L, H, w.N, D), "v_hist": (L, H, w.N, D),
    }
    if w.granularity == "token":
        shapes["q_score"] = (L, H, w.n_score_q, D)
    res = {k: torch.empty(s, dtype=dt) for k, s in shapes.items()}
    res["head_role"] = torch.empty((L, H), dtype=torch.uint8)
    res["static_mask"] = torch.empty((L, H, w.F * w.T if w.static_token_mask else w.F),
                                     dtype=torch.uint8)
    res["k_per_head"] = torch.empty((L, H), dtype=torch.int32)

    def one(l):
        arrs, role, mask, kph = _layer(w, w.seeds()[l])
        for k, a in arrs.items():
            res[k][l].copy_(torch.from_numpy(a))
        res["head_role"][l] = torch.from_numpy(role)
        res["static_mask"][l] = torch.from_numpy(mask)
        res["k_per_head"][l] = torch.from_numpy(kph)

    nthreads = threads or min(L, max(1, (os.cpu_count() or 1)))
    if nthreads <= 1 or L == 1:
        for l in range(L):
            one(l)
    else:
        with _cf.ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(one, range(L)))
    return res


def as_float64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a generated tensor for the fp64 oracle."""
    return t.to(torch.float64).numpy()


def sample_rows(n_rows: int, n_samples: int, seed: int) -> np.ndarray:
    """Sorted distinct query rows for sampled checks; always includes the
    first and the last row so the ragged tail tile is covered."""
    if n_samples >= n_rows:
        return np.arange(n_rows)
    rng = np.random.default_rng(seed)
    pick = rng.choice(n_rows, size=n_samples - 2, replace=False)
    return np.unique(np.concatenate([pick, [0, n_rows - 1]]))


def tile_rows(n_rows: int, seed: int, tile: int = 128, per_tile: int = 1) -> np.ndarray:
    """Sorted distinct query rows with ``per_tile`` random rows inside every
    ``tile``-row block (the last, ragged block included) plus the first and the
    last row, so that every query tile of a head is checked."""
    rng = np.random.default_rng(seed)
    picks = [np.array([0, n_rows - 1])]
    for start in range(0, n_rows, tile):
        stop = min(n_rows, start + tile)
        picks.append(rng.choice(np.arange(start, stop), size=min(per_tile, stop - start),
                                replace=False))
    return np.unique(np.concatenate(picks))


__all__: Sequence[str] = (
    "Workload", "WORKLOADS", "STATIC_FRAMES_18", "get", "scaled", "generate",
    "as_float64", "sample_rows", "tile_rows",
)


def random_kept(w: Workload, seed: int, n_keep: Optional[int] = None):
    """Seeded kept-frame lists for exercising the compaction and attention on
    their own: per (layer, head) an ascending random subset of the F history
    frames, padded with -1.  Its size is n_keep (default: a random count);
    head (0, 0) keeps nothing and, when there are two or more heads, head
    (0, 1) keeps every frame.  Returns (kept_idx int32 [L][H][F], kept_cnt
    int32 [L][H])."""
    rng = np.random.default_rng(seed)
    idx = np.full((w.L, w.H, w.F), -1, dtype=np.int32)
    cnt = np.zeros((w.L, w.H), dtype=np.int32)
    for l in range(w.L):
        for h in range(w.H):
            if (l, h) == (0, 0):
                c = 0
            elif (l, h) == (0, 1):
                c = w.F
            else:
                c = int(rng.integers(0, w.F + 1)) if n_keep is None else n_keep
            frames = np.sort(rng.choice(w.F, size=c, replace=False)) if c else np.zeros(0, int)
            idx[l, h, :c] = frames
            cnt[l, h] = c
    return torch.from_numpy(idx), torch.from_numpy(cnt)
