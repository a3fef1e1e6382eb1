"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test ties one oracle function to something other than itself: a closed
form, a library routine (torch's scaled_dot_product_attention), brute-force
enumeration, an invariant, or a figure the pages print (tests/golden).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import fkv_workloads as wl
from oracle import fkv_loops as loops
from oracle import fkv_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- segment mass

def _closed_form_inputs(a, c, T, D, scale, stride=1, filler=None):
    """Keys of frame f are c_f * u, query i is a_i * u, with |u| = 1, so
    z_ij = scale * a_i * c_f and mass_f = sum_i exp(s a_i c_f) / sum_g exp(s a_i c_g)."""
    u = np.ones(D) / math.sqrt(D)
    k_hist = np.concatenate([np.tile(cf * u, (T, 1)) for cf in c], axis=0)
    rows = []
    for i, ai in enumerate(a):
        rows.append(ai * u)
        if filler is not None and i < len(a) - 1:
            for _ in range(stride - 1):
                rows.append(filler * u)
    return np.array(rows), k_hist


def _closed_form_mass(a, c, scale):
    out = []
    for cf in c:
        tot = 0.0
        for ai in a:
            den = sum(math.exp(scale * ai * cg) for cg in c)
            tot += math.exp(scale * ai * cf) / den
        out.append(tot)
    return np.array(out)


def test_mass_closed_form():
    a, c, T, D, scale = [1.5, -0.8, 2.0], [0.3, -1.2, 2.5, 0.9], 3, 4, 0.7
    q, k = _closed_form_inputs(a, c, T, D, scale)
    got = orc.segment_mass(q, k, T, scale)
    np.testing.assert_allclose(got, _closed_form_mass(a, c, scale), rtol=1e-13, atol=0)


def test_mass_uses_only_strided_rows():
    """Reading: scoring queries are rows 0, s, 2s, ...  Rows in between carry a
    large filler that would dominate the closed form if they were used."""
    a, c, T, D, scale, s = [1.5, -0.8, 2.0, 0.4], [0.3, -1.2, 2.5], 2, 8, 0.5, 4
    q, k = _closed_form_inputs(a, c, T, D, scale, stride=s, filler=40.0)
    got = orc.segment_mass(orc.scoring_queries(q, s), k, T, scale)
    np.testing.assert_allclose(got, _closed_form_mass(a, c, scale), rtol=1e-13)


def test_mass_rows_sum_to_query_count():
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal((7, 16)), rng.standard_normal((5 * 9, 16))
    m = orc.segment_mass(q, k, 9, 0.25)
    assert abs(m.sum() - 7.0) < 1e-12
    assert np.all(m > 0)


def test_mass_zero_query_is_uniform():
    rng = np.random.default_rng(6)
    k = rng.standard_normal((6 * 4, 8))
    m = orc.segment_mass(np.zeros((3, 8)), k, 4, 0.35)
    np.testing.assert_allclose(m, np.full(6, 3 * 4 / 24), rtol=1e-14)


def test_mass_matches_loop_spelling():
    rng = np.random.default_rng(7)
    q, k = rng.standard_normal((5, 6)), rng.standard_normal((4 * 3, 6))
    np.testing.assert_allclose(orc.segment_mass(q, k, 3, 0.4),
                               loops.segment_mass(q.tolist(), k.tolist(), 3, 0.4), rtol=1e-13)


# ---------------------------------------------------------------- selection

def _brute_topk(scores, k):
    """Max-sum k-subset; among equal sums the lexicographically smallest."""
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(range(len(scores)), k):  # lexicographic order
        s = sum(scores[i] for i in sub)
        if s > best_sum:
            best, best_sum = sub, s
    return list(best)


@pytest.mark.parametrize("seed", range(40))
def test_topk_bruteforce(seed):
    rng = np.random.default_rng(100 + seed)
    F = int(rng.integers(2, 9))
    k = int(rng.integers(0, F + 1))
    # small integer scores make exact ties common
    scores = rng.integers(0, 3, size=F).astype(np.float64) if seed % 2 else rng.random(F)
    assert list(orc.top_k(scores, k)) == _brute_topk(list(scores), k)
    assert orc.top_k(scores, k).tolist() == loops.top_k(list(scores), k)


def test_topk_ties_lower_index_and_ascending():
    assert orc.top_k(np.array([1.0, 3.0, 3.0, 3.0, 0.5]), 2).tolist() == [1, 2]
    assert orc.top_k(np.array([2.0, 1.0, 2.0]), 2).tolist() == [0, 2]
    assert orc.top_k(np.array([5.0, 4.0]), 0).tolist() == []


def test_topk_18_choose_13_bruteforce():
    rng = np.random.default_rng(11)
    scores = rng.random(18)
    assert orc.top_k(scores, 13).tolist() == _brute_topk(list(scores), 13)


def test_static_keep_is_mask_order():
    mask = np.array([1, 0, 0, 1, 1, 0, 1], dtype=np.uint8)
    assert orc.static_keep(mask).tolist() == [0, 3, 4, 6]
    assert orc.static_keep(np.zeros(4, np.uint8)).tolist() == []


# ---------------------------------------------------------------- token variant

def test_phi_integer_inputs_exact():
    rng = np.random.default_rng(12)
    q = rng.integers(-4, 5, size=(6, 5)).astype(np.float64)
    k = rng.integers(-4, 5, size=(9, 5)).astype(np.float64)
    got = orc.participative_phi(q, k)
    assert got.tolist() == loops.phi(q.tolist(), k.tolist())
    # linearity: phi_j = (sum_r q_r) . k_j, exact on integers
    assert got.tolist() == (k @ q.sum(axis=0)).tolist()


def _brute_token_keep(phi, N, S, R, C):
    cands = list(range(S, N - R))
    best, best_sum = None, -math.inf
    for sub in itertools.combinations(cands, C):
        s = sum(phi[j - S] for j in sub)
        if s > best_sum:
            best, best_sum = sub, s
    return list(range(S)) + list(best) + list(range(N - R, N))


@pytest.mark.parametrize("seed", range(12))
def test_token_keep_bruteforce(seed):
    rng = np.random.default_rng(200 + seed)
    N, S, R = 11, int(rng.integers(0, 3)), int(rng.integers(0, 3))
    n_c = N - S - R
    C = int(rng.integers(0, n_c + 1))
    phi = rng.integers(-2, 3, size=n_c).astype(np.float64)
    assert orc.token_keep(phi, N, S, R, C).tolist() == _brute_token_keep(list(phi), N, S, R, C)


# ---------------------------------------------------------------- compaction

def test_compact_row_identity():
    T, F, D = 3, 5, 2
    hist = np.repeat(np.arange(F * T, dtype=np.float64)[:, None], D, axis=1)
    got = orc.compact(hist, np.array([1, 4]), T)
    assert got[:, 0].tolist() == [3, 4, 5, 12, 13, 14]
    assert orc.compact(hist, np.array([], dtype=np.int64), T).shape == (0, D)
    assert orc.compact(hist, np.array([0, 7, 9]), 1)[:, 1].tolist() == [0, 7, 9]


# ---------------------------------------------------------------- attention

def _sdpa(q, k, v, scale):
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    return torch.nn.functional.scaled_dot_product_attention(
        t(q), t(k), t(v), scale=scale)[0, 0].numpy()


def test_attention_equals_sdpa():
    rng = np.random.default_rng(13)
    q, k, v = rng.standard_normal((9, 16)), rng.standard_normal((20, 16)), rng.standard_normal((20, 8))
    np.testing.assert_allclose(orc.attention(q, k, v, 0.3), _sdpa(q, k, v, 0.3), rtol=0, atol=1e-12)


def test_attention_constant_values_and_dominant_key():
    rng = np.random.default_rng(14)
    q, k = rng.standard_normal((4, 8)), rng.standard_normal((10, 8))
    v = np.tile(np.arange(8.0), (10, 1))
    np.testing.assert_allclose(orc.attention(q, k, v, 0.5), np.tile(np.arange(8.0), (4, 1)), atol=1e-13)
    k2 = k.copy()
    k2[6] = 60.0 * q[0] / np.linalg.norm(q[0])
    v2 = rng.standard_normal((10, 8))
    o = orc.attention(q[:1], k2, v2, 1.0)
    np.testing.assert_allclose(o[0], v2[6], atol=1e-9)


def _tiny_f64(w):
    t = wl.generate(w)
    return {k: (wl.as_float64(v) if v.is_floating_point() else v.numpy()) for k, v in t.items()}


def test_step_without_pruning_is_full_attention():
    """0% pruning (every frame kept) reproduces full attention over history + chunk."""
    w = wl.get("tiny")
    x = _tiny_f64(w)
    mask = np.ones_like(x["static_mask"])
    kph = np.full_like(x["k_per_head"], w.F)
    res = orc.step(x["q_cur"], x["k_cur"], x["v_cur"], x["k_hist"], x["v_hist"],
                   x["head_role"], mask, kph, T=w.T, granularity="frame", scale=w.scale)
    for h in range(w.H):
        assert res["kept"][(0, h)].tolist() == list(range(w.F))
        kk = np.concatenate([x["k_hist"][0, h], x["k_cur"][0, h]])
        vv = np.concatenate([x["v_hist"][0, h], x["v_cur"][0, h]])
        np.testing.assert_allclose(res["out"][(0, h)], _sdpa(x["q_cur"][0, h], kk, vv, w.scale),
                                   rtol=0, atol=1e-12)


def test_step_pruned_equals_sdpa_over_selected_keys():
    w = wl.get("tiny")
    x = _tiny_f64(w)
    res = orc.step(x["q_cur"], x["k_cur"], x["v_cur"], x["k_hist"], x["v_hist"],
                   x["head_role"], x["static_mask"], x["k_per_head"],
                   T=w.T, granularity="frame", scale=w.scale)
    for h in range(w.H):
        kept = res["kept"][(0, h)]
        assert len(kept) == 2
        if x["head_role"][0, h] == 0:
            assert kept.tolist() == [0, 5]
        idx = torch.from_numpy((kept[:, None] * w.T + np.arange(w.T)[None]).reshape(-1))
        kk = torch.cat([torch.from_numpy(x["k_hist"][0, h]).index_select(0, idx),
                        torch.from_numpy(x["k_cur"][0, h])]).numpy()
        vv = torch.cat([torch.from_numpy(x["v_hist"][0, h]).index_select(0, idx),
                        torch.from_numpy(x["v_cur"][0, h])]).numpy()
        np.testing.assert_allclose(res["out"][(0, h)], _sdpa(x["q_cur"][0, h], kk, vv, w.scale),
                                   rtol=0, atol=1e-12)


def test_step_matches_loop_spelling_on_tiny():
    w = wl.get("tiny")
    x = _tiny_f64(w)
    res = orc.step(x["q_cur"], x["k_cur"], x["v_cur"], x["k_hist"], x["v_hist"],
                   x["head_role"], x["static_mask"], x["k_per_head"],
                   T=w.T, granularity="frame", scale=w.scale)
    for h in range(w.H):
        kept, mass, outs = loops.step_head(
            x["q_cur"][0, h].tolist(), x["k_cur"][0, h].tolist(), x["v_cur"][0, h].tolist(),
            x["k_hist"][0, h].tolist(), x["v_hist"][0, h].tolist(),
            dynamic=bool(x["head_role"][0, h]), mask_row=x["static_mask"][0, h].tolist(),
            k=int(x["k_per_head"][0, h]), T=w.T, scale=w.scale)
        assert kept == res["kept"][(0, h)].tolist()
        if mass is not None:
            np.testing.assert_allclose(res["score"][(0, h)], mass, rtol=1e-12)
        np.testing.assert_allclose(res["out"][(0, h)], np.array(outs), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- page figures

def test_kept_fraction_matches_page_figures():
    g = json.load(open(os.path.join(GOLDEN, "page_figures.json")))
    w = wl.get("480p")
    # every head keeps 13 of 18 history frames (static mask or top-13)
    assert len(w.static_frames) == w.k_dynamic == 13
    reduction = 1.0 - 13 / 18
    assert abs(reduction - g["cache_reduction"]["value"]) < 0.05  # "about 30%"
    t = wl.get("token14b")
    window = (t.F + t.Fc) * t.T
    budget = t.keep_tokens + t.sink_tokens + t.recent_tokens  # C = N - S - R
    lo, hi = g["budget_fraction_of_window"]["min"], g["budget_fraction_of_window"]["max"]
    assert lo <= budget / window <= hi
    assert t.keep_tokens == 15210 and budget == 24570
    # whole-window reduction of the token variant vs the page's ~24%
    assert abs((window - budget) / window - g["deep_forcing_memory_reduction"]["value"]) < 0.02


def test_token_step_scores_the_candidate_rows():
    """Token variant on a small integer case: phi_j = R * sum_d k_j,d exactly when
    every scoring query is all-ones; the kept set is brute-forced from that."""
    rng = np.random.default_rng(15)
    H, N, D, S, R, C, Lq, Rq = 2, 12, 4, 2, 3, 4, 5, 3
    k_hist = rng.integers(-3, 4, size=(1, H, N, D)).astype(np.float64)
    v_hist = rng.standard_normal((1, H, N, D))
    q_cur, k_cur, v_cur = (rng.standard_normal((1, H, Lq, D)) for _ in range(3))
    q_score = np.ones((1, H, Rq, D))
    res = orc.step(q_cur, k_cur, v_cur, k_hist, v_hist, np.ones((1, H), np.uint8),
                   np.zeros((1, H, 1), np.uint8), np.full((1, H), C), T=1,
                   granularity="token", scale=0.5, q_score=q_score, sink=S, recent=R)
    for h in range(H):
        phi = [Rq * k_hist[0, h, j].sum() for j in range(S, N - R)]
        np.testing.assert_array_equal(res["score"][(0, h)], phi)
        kept = _brute_token_keep(phi, N, S, R, C)
        assert res["kept"][(0, h)].tolist() == kept
        kk = np.concatenate([k_hist[0, h][kept], k_cur[0, h]])
        vv = np.concatenate([v_hist[0, h][kept], v_cur[0, h]])
        np.testing.assert_allclose(res["out"][(0, h)], _sdpa(q_cur[0, h], kk, vv, 0.5), atol=1e-12)


def test_empty_history_keeps_nothing():
    assert orc.segment_mass(np.ones((2, 4)), np.zeros((0, 4)), 3, 0.5).shape == (0,)
    assert orc.top_k(np.zeros(0), 0).tolist() == []


def test_advance_keeps_the_most_recent_segments_then_the_chunk():
    T, D = 2, 3
    comp = np.repeat(np.arange(10, dtype=np.float64)[:, None], D, axis=1)  # 5 kept frames
    chunk = np.repeat(np.arange(100, 104, dtype=np.float64)[:, None], D, axis=1)  # 2 frames
    got = orc.advance(comp, 5, T, chunk, out_segments=5)   # keep 3 kept frames + 2 chunk
    assert got[:, 0].tolist() == [4, 5, 6, 7, 8, 9, 100, 101, 102, 103]
    got = orc.advance(comp, 5, T, chunk, out_segments=2)   # chunk only
    assert got[:, 0].tolist() == [100, 101, 102, 103]
    got = orc.advance(comp, 4, 1, chunk[:1], out_segments=3)  # token mode: last 2 of 4 kept
    assert got[:, 2].tolist() == [2, 3, 100]
    with pytest.raises(AssertionError):
        orc.advance(comp, 2, T, chunk, out_segments=6)


def test_mass_with_chunk_in_the_normaliser_closed_form():
    """Frame keys c_f * u, chunk keys c_x * u (Lq of them): the normaliser of row
    i gains Lq * exp(s a_i c_x); masses are still per history frame."""
    a, c, cx, T, Lq, D, scale = [1.5, -0.8, 2.0], [0.3, -1.2, 2.5], 0.7, 4, 6, 8, 0.6
    q, k = _closed_form_inputs(a, c, T, D, scale)
    u = np.ones(D) / math.sqrt(D)
    kc = np.tile(cx * u, (Lq, 1))
    got = orc.segment_mass(q, k, T, scale, k_chunk=kc)
    exp = []
    for cf in c:
        tot = 0.0
        for ai in a:
            den = T * sum(math.exp(scale * ai * cg) for cg in c) + Lq * math.exp(scale * ai * cx)
            tot += T * math.exp(scale * ai * cf) / den
        exp.append(tot)
    np.testing.assert_allclose(got, exp, rtol=1e-13)
    assert got.sum() < len(a)  # part of each row's mass now sits on the chunk


def test_token_static_mask_keeps_tokens_and_expands_frames():
    T = 3
    mask = np.zeros(12, np.uint8)
    mask[[0, 2, 5, 11]] = 1
    kept, sc = orc.head_keep(granularity="frame", dynamic=False, mask_row=mask, k=0,
                             q_cur=np.zeros((2, 4)), k_hist=np.zeros((12, 4)), T=T, scale=1.0,
                             token_static_mask=True)
    assert kept.tolist() == [0, 2, 5, 11] and sc is None
    assert orc.frames_to_tokens(np.array([1, 3]), T).tolist() == [3, 4, 5, 9, 10, 11]
    rng = np.random.default_rng(16)
    q, k = rng.standard_normal((3, 4)), rng.standard_normal((12, 4))
    kept, mass = orc.head_keep(granularity="frame", dynamic=True, mask_row=mask, k=2, q_cur=q,
                               k_hist=k, T=T, scale=0.5, token_static_mask=True)
    assert kept.tolist() == orc.frames_to_tokens(orc.top_k(mass, 2), T).tolist()


def test_rope_shift_rotation_identities():
    rng = np.random.default_rng(17)
    k = rng.standard_normal((5, 8))
    om = np.array([0.5, 1.25, 3.0])
    # rotating by a then by b is rotating by a + b; by -d undoes d
    np.testing.assert_allclose(orc.rope_shift(orc.rope_shift(k, om, 2.0), om, 3.0),
                               orc.rope_shift(k, om, 5.0), atol=1e-12)
    np.testing.assert_allclose(orc.rope_shift(orc.rope_shift(k, om, 4.0), om, -4.0), k, atol=1e-12)
    # a quarter turn maps (x0, x1) to (-x1, x0); dims past the band are untouched
    q = orc.rope_shift(k, np.array([math.pi / 2]), 1.0)
    np.testing.assert_allclose(q[:, 0], -k[:, 1], atol=1e-15)
    np.testing.assert_allclose(q[:, 1], k[:, 0], atol=1e-15)
    assert np.array_equal(q[:, 2:], k[:, 2:])
    # pair norms are preserved
    r = orc.rope_shift(k, om, 7.0)
    for i in range(3):
        np.testing.assert_allclose(np.hypot(r[:, 2 * i], r[:, 2 * i + 1]),
                                   np.hypot(k[:, 2 * i], k[:, 2 * i + 1]), rtol=1e-13)
    # delta 0 (a frame that keeps its place) is the identity
    np.testing.assert_allclose(orc.rope_shift(k, om, 0.0), k, atol=0)


def test_compact_repositioned_closes_the_gaps():
    T, F, D = 2, 6, 4
    k = np.arange(F * T * D, dtype=np.float64).reshape(F * T, D)
    om = np.array([0.3])
    got = orc.compact_repositioned(k, np.array([1, 4, 5]), T, F, om)
    # frames 1, 4, 5 move to 3, 4, 5: deltas 2, 0, 0
    np.testing.assert_allclose(got[:2], orc.rope_shift(k[2:4], om, 2.0), atol=1e-12)
    assert np.array_equal(got[2:], k[8:12])
