"""The step at the edges of its size limits, against the oracle: the largest
frame count (1024 history frames: the frame selection's 1024-thread CTA, 1024
frame entries per scoring row), more token candidates than the token
selection caches in shared memory (its uncached radix path), and a thousand
(layer, head) pairs in one call."""
import numpy as np
import pytest

import fkv_workloads as wl
from tests import parity

pytestmark = pytest.mark.gpu


def test_max_frames(cuda_device):
    # 1024 frames of 8 tokens; dynamic heads keep 700 of them
    w = wl.scaled(wl.get("480p"), name="max_frames", H=2, T=8, F=1024, Fc=2, n_static=1,
                  static_frames=tuple(range(0, 1024, 3)), k_dynamic=700, score_stride=1, seed=71)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    st = parity.check_step(w, x, res)
    print("max frames", st)
    assert (res["kept_cnt"][0] == np.array([len(range(0, 1024, 3)), 700])).all() or \
           (res["kept_cnt"][0] == np.array([700, len(range(0, 1024, 3))])).all()


def test_token_selection_uncached_path(cuda_device):
    # 60000 history tokens, 56000 candidates: above the 40960 keys a selection
    # CTA caches in shared memory, so every radix pass re-reads the scores
    w = wl.scaled(wl.get("token14b"), name="token_uncached", H=2, T=2000, F=30, Fc=1,
                  sink_tokens=2000, recent_tokens=2000, keep_tokens=40000, n_score_q=64, seed=72)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    rows = wl.sample_rows(w.Fc * w.T, 24, seed=3)
    st = parity.check_step(w, x, res, rows=rows)
    print("token uncached", st)
    assert (res["kept_cnt"] == 2000 + 40000 + 2000).all()


def test_thousand_heads(cuda_device):
    # L*H = 1024 heads of small frames in one call (grids over heads, dynamic
    # head counting in the scoring kernel, per-head selection)
    w = wl.scaled(wl.get("480p"), name="many_heads", L=4, H=256, T=64, F=5, Fc=1, n_static=128,
                  static_frames=(0, 2, 4), k_dynamic=3, score_stride=2, seed=73,
                  layer_seeds=(1, 2, 3, 4))
    x = wl.generate(w)
    res = parity.run_step(w, x)
    heads = [(l, h) for l in range(4) for h in (0, 1, 127, 128, 200, 255)]
    st = parity.check_step(w, x, res, heads=heads)
    print("thousand heads", st)
    assert (res["kept_cnt"] == 3).all()
