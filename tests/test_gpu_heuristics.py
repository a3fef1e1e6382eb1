"""Comparison selectors (uniform eviction, random drop) on the GPU against the
oracle: kept lists are integers and must match exactly; the random
priorities are 24-bit grid values and must match bit for bit.

Forcing-KV (ai-feeds.com/i/paper/2605.09681), "与基线对比及工程启示", first
item; token granularity: Deep Forcing (bxzpzcl.cn/news/2125000), section 3.1.
"""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_heuristics as fh

pytestmark = pytest.mark.gpu


def _run(p, policy, seed, k):
    o = fkv.allocate(p)
    kept_idx, kept_cnt, seg = o["kept_idx"], o["kept_cnt"], o["seg_score"]
    fkv.select_heuristic(p, policy, seed, k.cuda(), kept_idx, kept_cnt, o["ws"],
                         seg_score=seg if policy == "random" else None)
    assert fkv.read_status(o["ws"])[0] == 0
    return kept_idx.cpu().numpy(), kept_cnt.cpu().numpy(), seg.cpu().numpy()


@pytest.mark.parametrize("policy", ["uniform", "random"])
@pytest.mark.parametrize("seed", [0, 2**63 + 12345])
def test_frame_mode_exact(cuda_device, policy, seed):
    w = wl.get("480p")
    p = fkv.params_for(w)
    rng = np.random.default_rng(5)
    k = torch.from_numpy(rng.integers(0, w.F + 1, size=(w.L, w.H)).astype(np.int32))
    k[0, 0], k[0, 1], k[0, 2] = 0, w.F, 13
    idx, cnt, seg = _run(p, policy, seed, k)
    for l in range(w.L):
        for h in range(w.H):
            lh = l * w.H + h
            want = fh.head_keep(policy, granularity="frame", seed=seed, lh=lh, k=int(k[l, h]), F=w.F)
            assert cnt[l, h] == len(want) and np.array_equal(idx[l, h, :len(want)], want), (l, h)
            if policy == "random":
                u = fh.priorities(seed, lh, w.F).astype(np.float32)
                assert np.array_equal(seg[l, h].view(np.uint32), u.view(np.uint32))


@pytest.mark.parametrize("policy", ["uniform", "random"])
def test_token_mode_exact(cuda_device, policy):
    w = wl.scaled(wl.get("token14b"), name="heur_tok", H=4, T=96, F=10, sink_tokens=192,
                  recent_tokens=96, keep_tokens=300, n_score_q=96)
    n_c = w.N - w.sink_tokens - w.recent_tokens
    p = fkv.params_for(w)
    k = torch.tensor([[0, n_c, n_c // 2, 7]], dtype=torch.int32)
    idx, cnt, _ = _run(p, policy, 77, k)
    for h in range(w.H):
        want = fh.head_keep(policy, granularity="token", seed=77, lh=h, k=int(k[0, h]), N=w.N,
                            sink=w.sink_tokens, recent=w.recent_tokens)
        assert cnt[0, h] == len(want) and np.array_equal(idx[0, h, :len(want)], want), h


def test_token14b_random_two_heads(cuda_device):
    w = wl.get("token14b")
    p = fkv.params_for(w)
    n_c = w.N - w.sink_tokens - w.recent_tokens
    k = torch.full((w.L, w.H), w.keep_tokens, dtype=torch.int32)
    idx, cnt, seg = _run(p, "random", 2024, k)
    for h in (0, w.H - 1):  # the oracle's pure-Python Philox bounds how many heads it checks
        want = fh.head_keep("random", granularity="token", seed=2024, lh=h, k=w.keep_tokens, N=w.N,
                            sink=w.sink_tokens, recent=w.recent_tokens)
        assert cnt[0, h] == len(want) and np.array_equal(idx[0, h, :len(want)], want), h
    assert np.all(cnt == w.sink_tokens + w.keep_tokens + w.recent_tokens)
    assert seg.shape[-1] == n_c
