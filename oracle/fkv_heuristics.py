"""Comparison selectors of the Forcing-KV page -- TEST INFRASTRUCTURE ONLY.

The Forcing-KV page compares its head-wise selection with uniform eviction
and random dropping at the same compression ratio (Forcing-KV,
ai-feeds.com/i/paper/2605.09681, "与基线对比及工程启示", first item) without
defining either.  The reading implemented here keeps the budget of every head
(k_per_head: k frames, or C candidate tokens) and ignores head roles, since a
baseline compresses every head the same way:

  * uniform eviction: of n segments keep those at floor(i * n / k), i < k
    (evenly spaced, the first segment always kept);
  * random drop: keep the k segments of largest priority u(seed; lh, s), ties
    to the lower index, with u the first 64-bit word of Philox4x64-10 at
    counter (s, lh, 0, 0) and key (seed, 0), its top 24 bits scaled to [0, 1).

Token granularity (Deep Forcing, bxzpzcl.cn/news/2125000, section 3.1): the
sink [0, S) and recent [N - R, N) tokens are kept whole and the selectors
apply to the n = N - S - R candidates between them.

Philox4x64-10 follows its published definition (Salmon, Moraes, Dror and Shaw,
"Parallel random numbers: as easy as 1, 2, 3", SC 2011): ten rounds of two
64 x 64 -> 128-bit products with the Weyl-sequence key schedule.
"""
from __future__ import annotations

from typing import Sequence, Tuple

import numpy as np

_MASK64 = (1 << 64) - 1
# Philox4x64 round multipliers and key increments (Salmon et al., 2011).
_M0, _M1 = 0xD2E7470EE14C6C93, 0xCA5A826395121157
_W0, _W1 = 0x9E3779B97F4A7C15, 0xBB67AE8584CAA73B


def philox4x64_10(ctr: Sequence[int], key: Sequence[int]) -> Tuple[int, int, int, int]:
    """Philox4x64 with 10 rounds on Python integers."""
    c0, c1, c2, c3 = (int(v) & _MASK64 for v in ctr)
    k0, k1 = (int(v) & _MASK64 for v in key)
    for r in range(10):
        if r:
            k0 = (k0 + _W0) & _MASK64
            k1 = (k1 + _W1) & _MASK64
        p0 = _M0 * c0
        p1 = _M1 * c2
        hi0, lo0 = p0 >> 64, p0 & _MASK64
        hi1, lo1 = p1 >> 64, p1 & _MASK64
        c0, c1, c2, c3 = hi1 ^ c1 ^ k0, lo1, hi0 ^ c3 ^ k1, lo0
    return c0, c1, c2, c3


def priority(seed: int, lh: int, s: int) -> float:
    """u(seed; lh, s) in [0, 1): top 24 bits of Philox4x64-10's first word."""
    w0 = philox4x64_10((s, lh, 0, 0), (seed, 0))[0]
    return (w0 >> 40) * 2.0 ** -24


def priorities(seed: int, lh: int, n: int) -> np.ndarray:
    """u(seed; lh, s) for s < n."""
    return np.array([priority(seed, lh, s) for s in range(n)], dtype=np.float64)


def uniform_keep(n: int, k: int) -> np.ndarray:
    """Uniform eviction: segments floor(i * n / k), i < k, ascending (0 <= k <= n)."""
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    return np.array([(i * n) // k for i in range(k)], dtype=np.int64)


def random_keep(seed: int, lh: int, n: int, k: int) -> np.ndarray:
    """Random drop: the k segments of largest priority, ties to the lower index, ascending."""
    if k <= 0:
        return np.zeros(0, dtype=np.int64)
    u = priorities(seed, lh, n)
    order = sorted(range(n), key=lambda s: (-u[s], s))
    return np.array(sorted(order[:k]), dtype=np.int64)


def head_keep(policy: str, *, granularity: str, seed: int, lh: int, k: int, F: int = 0,
              N: int = 0, sink: int = 0, recent: int = 0) -> np.ndarray:
    """Kept list of head lh under a comparison selector: frames (frame mode) or
    token indices (token mode, sink and recent included), ascending."""
    pick = uniform_keep if policy == "uniform" else None
    if granularity == "frame":
        return uniform_keep(F, k) if pick else random_keep(seed, lh, F, k)
    n_c = N - sink - recent
    cand = uniform_keep(n_c, k) if pick else random_keep(seed, lh, n_c, k)
    return np.concatenate([np.arange(sink), sink + cand, np.arange(N - recent, N)]).astype(np.int64)
