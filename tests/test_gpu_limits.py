"""The step at the edges of its size limits, against the oracle: the largest
frame count (1024 history frames: the frame selection's 1024-thread CTA, 1024
frame entries per scoring row), more token candidates than the token
selection caches in shared memory (its uncached radix path), the cached path
with and without the first pass's candidate list (and a list that overflows),
and a thousand (layer, head) pairs in one call."""
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


def test_token_selection_cached_without_candidate_list(cuda_device):
    # 30000 candidates: cached in shared memory, but above the 24576 keys for
    # which the selection also keeps a candidate list after its first pass
    w = wl.scaled(wl.get("token14b"), name="token_cached_nolist", H=2, T=1000, F=32, Fc=1,
                  sink_tokens=1000, recent_tokens=1000, keep_tokens=21000, n_score_q=64,
                  seed=74)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    rows = wl.sample_rows(w.Fc * w.T, 24, seed=4)
    st = parity.check_step(w, x, res, rows=rows)
    print("token cached, no candidate list", st)
    assert (res["kept_cnt"] == 1000 + 21000 + 1000).all()


def test_token_selection_candidate_list_overflow(cuda_device):
    # 20000 candidates with one key row repeated: every score is equal, so all
    # 20000 share the first pass's bin, more than the 16384-entry candidate
    # list holds; the selection falls back to scanning every key and keeps
    # the lowest indices (ties in index order)
    w = wl.scaled(wl.get("token14b"), name="token_list_overflow", H=2, T=1000, F=22, Fc=1,
                  sink_tokens=1000, recent_tokens=1000, keep_tokens=12000, n_score_q=64,
                  seed=75)
    x = wl.generate(w)
    c0, c1 = w.sink_tokens, w.N - w.recent_tokens
    x["k_hist"][:, :, c0:c1] = x["k_hist"][:, :, c0:c0 + 1]
    res = parity.run_step(w, x)
    rows = wl.sample_rows(w.Fc * w.T, 24, seed=5)
    st = parity.check_step(w, x, res, rows=rows)
    print("token candidate list overflow", st)
    for h in range(w.H):
        kept = parity.gpu_kept(res, 0, h)
        assert kept[c0:c0 + 12000].tolist() == list(range(c0, c0 + 12000))


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
