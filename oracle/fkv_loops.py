"""Pure-Python loop spelling of the chunk step (test infrastructure, tiny inputs).

A second, independent implementation of the same definitions as
``fkv_oracle`` using only ``math`` and Python lists: used on the tiny workload
to cross-check the numpy oracle.  Sources as in ``fkv_oracle``: Forcing-KV
(ai-feeds.com/i/paper/2605.09681) "关键模块" 2-3 and "输出与工程收益";
Deep Forcing (bxzpzcl.cn/news/2125000) section 3.1.
"""
from __future__ import annotations

import math
from typing import List, Sequence


def dot(a: Sequence[float], b: Sequence[float]) -> float:
    s = 0.0
    for x, y in zip(a, b):
        s += float(x) * float(y)
    return s


def segment_mass(q_rows, k_hist, T: int, scale: float) -> List[float]:
    """mass_f = sum over scoring rows of the softmax mass on frame f's keys."""
    N = len(k_hist)
    F = N // T
    mass = [0.0] * F
    for q in q_rows:
        z = [scale * dot(q, k) for k in k_hist]
        m = max(z)
        e = [math.exp(v - m) for v in z]
        tot = sum(e)
        for j in range(N):
            mass[j // T] += e[j] / tot
    return mass


def top_k(scores: Sequence[float], k: int) -> List[int]:
    """Repeatedly take the best remaining index (strictly greater wins, so the
    lower index wins a tie); return the chosen set ascending."""
    left = list(range(len(scores)))
    chosen = []
    for _ in range(k):
        best = left[0]
        for i in left[1:]:
            if scores[i] > scores[best]:
                best = i
        chosen.append(best)
        left.remove(best)
    return sorted(chosen)


def phi(q_score, k_cand) -> List[float]:
    """phi_j = sum_r q_r . k_j, as a double loop."""
    return [sum(dot(q, k) for q in q_score) for k in k_cand]


def attention_row(q, keys, values, scale: float) -> List[float]:
    z = [scale * dot(q, k) for k in keys]
    m = max(z)
    e = [math.exp(v - m) for v in z]
    tot = sum(e)
    D = len(values[0])
    o = [0.0] * D
    for w, v in zip(e, values):
        for d in range(D):
            o[d] += w * float(v[d])
    return [x / tot for x in o]


def step_head(q_cur, k_cur, v_cur, k_hist, v_hist, *, dynamic: bool, mask_row, k: int,
              T: int, scale: float, score_stride: int = 1):
    """Frame-granular step for one head: (kept frames, mass or None, outputs)."""
    if dynamic:
        mass = segment_mass(q_cur[0::score_stride], k_hist, T, scale)
        kept = top_k(mass, k)
    else:
        mass = None
        kept = [f for f in range(len(mask_row)) if mask_row[f]]
    keys, vals = [], []
    for f in kept:
        keys.extend(k_hist[f * T:(f + 1) * T])
        vals.extend(v_hist[f * T:(f + 1) * T])
    keys.extend(k_cur)
    vals.extend(v_cur)
    outs = [attention_row(q, keys, vals, scale) for q in q_cur]
    return kept, mass, outs
