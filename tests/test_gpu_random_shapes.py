"""Randomly shaped small steps against the oracle.

A fixed-seed sweep over sizes the hand-written cases do not enumerate: frame
lengths from 1 to 300 tokens (ragged 128-key tiles of every size), 0 to 9
history frames, 1 to 3 chunk frames, 1 to 6 heads with any static/dynamic
split, any budget up to F and scoring strides from 1 to 8 -- so odd and even
attention block counts, empty histories, one-block units and tiles straddling
the compressed/chunk boundary all occur.  A few token-mode cases draw sink,
recent and candidate counts the same way.  The configurations are drawn once
at import, so test ids are stable."""
import numpy as np
import pytest

import fkv_workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu


def _frame_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        H = int(rng.integers(1, 7))
        T = int(rng.integers(1, 301))
        F = int(rng.integers(0, 10))
        Fc = int(rng.integers(1, 4))
        n_static = int(rng.integers(0, H + 1))
        k = int(rng.integers(0, F + 1))
        n_frames = int(rng.integers(0, F + 1))
        frames = tuple(sorted(int(f) for f in rng.choice(F, size=n_frames, replace=False))) if F else ()
        stride = int(rng.integers(1, 9))
        fp32 = i % 4 == 3
        cases.append(dict(name=f"rand_frame_{i}", H=H, T=T, F=F, Fc=Fc, n_static=n_static,
                          static_frames=frames, k_dynamic=k, score_stride=stride,
                          dtype="fp32" if fp32 else "bf16", D=64 if fp32 else 128,
                          seed=100 + i))
    return cases


def _token_cases(n, seed):
    rng = np.random.default_rng(seed)
    cases = []
    for i in range(n):
        H = int(rng.integers(1, 4))
        T = int(rng.integers(8, 129))
        F = int(rng.integers(3, 10))
        Fc = int(rng.integers(1, 3))
        N = F * T
        sink = int(rng.integers(0, T + 1))
        recent = int(rng.integers(0, T + 1))
        cand = N - sink - recent
        keep = int(rng.integers(0, cand + 1))
        n_score_q = int(rng.integers(1, T + 1))
        cases.append(dict(name=f"rand_token_{i}", H=H, T=T, F=F, Fc=Fc, sink_tokens=sink,
                          recent_tokens=recent, keep_tokens=keep, n_score_q=n_score_q,
                          seed=200 + i))
    return cases


FRAME_CASES = _frame_cases(12, seed=2026)
TOKEN_CASES = _token_cases(3, seed=2027)


@pytest.mark.parametrize("case", FRAME_CASES, ids=[c["name"] for c in FRAME_CASES])
def test_random_frame_step(cuda_device, case):
    w = wl.scaled(wl.get("480p"), **case)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)


@pytest.mark.parametrize("case", TOKEN_CASES, ids=[c["name"] for c in TOKEN_CASES])
def test_random_token_step(cuda_device, case):
    w = wl.scaled(wl.get("token14b"), **case)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)
