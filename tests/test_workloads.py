"""The seeded generators: shapes, determinism and the stated structure."""
import numpy as np
import torch

import fkv_workloads as wl


def test_tiny_shapes_roles_and_determinism():
    w = wl.get("tiny")
    a, b = wl.generate(w), wl.generate(w)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["q_cur"].shape == (1, 4, 32, 64) and a["q_cur"].dtype == torch.float32
    assert a["k_hist"].shape == (1, 4, 192, 64)
    assert a["head_role"].tolist() == [[0, 0, 1, 1]]
    assert a["static_mask"][0, 0].tolist() == [1, 0, 0, 0, 0, 1]
    assert a["k_per_head"].tolist() == [[0, 0, 2, 2]]


def test_video_recipe_small_and_thread_independent():
    w = wl.scaled(wl.get("480p"), L=3, T=16, layer_seeds=(5, 6, 7))
    a, b = wl.generate(w, threads=1), wl.generate(w, threads=3)
    for k in a:
        assert torch.equal(a[k], b[k]), k
    assert a["k_hist"].dtype == torch.bfloat16
    role = a["head_role"]
    assert (role.sum(dim=1) == 6).all()
    m = a["static_mask"]
    for l in range(3):
        for h in range(12):
            if role[l, h] == 0:
                assert m[l, h].nonzero().flatten().tolist() == list(wl.STATIC_FRAMES_18)
            else:
                assert m[l, h].sum() == 0 and a["k_per_head"][l, h] == 13
    # frames differ: per-frame means of history K are spread out
    k = a["k_hist"][0, 0].float().reshape(18, 16, 128).mean(dim=1)
    assert k.std(dim=0).mean() > 0.3


def test_token_workload_budget():
    w = wl.get("token14b")
    assert w.n_segments == 18720 and w.keep_tokens == 15210
    s = wl.scaled(w, H=2, T=8, n_score_q=8, sink_tokens=24, recent_tokens=24, keep_tokens=50)
    x = wl.generate(s)
    assert x["q_score"].shape == (1, 2, 8, 128)
    assert x["head_role"].tolist() == [[1, 1]]
    assert x["k_per_head"].tolist() == [[50, 50]]


def test_sample_rows_covers_ends():
    r = wl.sample_rows(4680, 64, 3)
    assert r[0] == 0 and r[-1] == 4679 and len(np.unique(r)) == len(r)


def test_tile_rows_hit_every_tile_and_both_ends():
    for n in (4680, 24480, 128, 129, 37):
        r = wl.tile_rows(n, seed=5)
        assert r[0] == 0 and r[-1] == n - 1 and np.all(np.diff(r) > 0)
        assert set(range(-(-n // 128))) <= set((r // 128).tolist())
