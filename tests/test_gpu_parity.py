"""Parity of the CUDA path with the fp64 oracle on every workload.

Small cases and the 480P layer are compared on every output element (every
query row of every head).  The larger workloads (1080P, the 30-layer batch,
the 14B token variant), run in the launch configuration the benchmark times,
are compared on every score, kept index and compacted row of every head, and
on attention rows that include a random row of every 128-query tile plus the
first and last row, so that every work unit of the persistent attention
kernel (one query tile of one head) carries a checked row."""
import numpy as np
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from oracle import fkv_oracle as orc
from tests import parity

pytestmark = pytest.mark.gpu


def test_tiny_fp32_full(cuda_device):
    w = wl.get("tiny")
    x = wl.generate(w)
    res = parity.run_step(w, x)
    st = parity.check_step(w, x, res)
    assert st["sel_tie"] == 0


def test_tiny_fp32_entry_points_one_by_one(cuda_device):
    """Each entry point alone, fed the previous step's oracle-checked output."""
    w = wl.get("tiny")
    x = wl.generate(w)
    p = fkv.params_for(w)
    d = parity.upload(x)
    o = fkv.allocate(p)
    fkv.score_segments(p, d["q_cur"], None, d["k_hist"], d["head_role"], o["seg_score"], o["ws"])
    fkv.select_topk(p, o["seg_score"], d["head_role"], d["static_mask"], d["k_per_head"],
                    o["kept_idx"], o["kept_cnt"], o["ws"])
    fkv.compact_gather(p, d["k_hist"], d["v_hist"], o["kept_idx"], o["kept_cnt"], o["k_comp"],
                       o["v_comp"], o["ws"])
    fkv.attend_compressed(p, d["q_cur"], d["k_cur"], d["v_cur"], o["k_comp"], o["v_comp"],
                          o["kept_cnt"], o["out"], o["ws"])
    res = {k: v.cpu() for k, v in o.items() if k != "ws"}
    res["status"] = fkv.read_status(o["ws"])
    parity.check_step(w, x, res)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_small_multi_tile_ragged(cuda_device, dtype):
    """Several tiles with ragged tails everywhere: T = 200, stride 3."""
    w = wl.scaled(wl.get("480p"), name=f"small_{dtype}", H=4, T=200, F=7, Fc=2, n_static=2,
                  static_frames=(0, 3, 6), k_dynamic=4, score_stride=3, dtype=dtype, seed=21)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)


def test_small_token_variant(cuda_device):
    w = wl.scaled(wl.get("token14b"), name="small_token", H=3, T=64, F=9, Fc=2, n_score_q=64,
                  sink_tokens=128, recent_tokens=128, keep_tokens=200, seed=22)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)


def _full(name):
    w = wl.get(name)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    return w, x, res


def test_480p_full_size_every_row(cuda_device):
    w, x, res = _full("480p")
    st = parity.check_step(w, x, res)  # every head, every query row
    print("480p", st)


def test_1080p_full_size(cuda_device):
    w, x, res = _full("1080p")
    rows = wl.tile_rows(w.Lq, seed=7)
    assert len(rows) >= -(-w.Lq // 128)
    st = parity.check_step(w, x, res, rows=rows)
    print("1080p", st)


def test_token14b_full_size(cuda_device):
    w, x, res = _full("token14b")
    st = parity.check_step(w, x, res, rows=wl.tile_rows(w.Lq, seed=7))
    print("token14b", st)
    # every head keeps S + C + R tokens
    assert (res["kept_cnt"] == w.sink_tokens + w.keep_tokens + w.recent_tokens).all()


def test_480p_30_layers(cuda_device):
    w, x, res = _full("480p_30layer")
    assert (res["kept_cnt"] == 13).all()
    st = parity.check_step(w, x, res, rows=wl.tile_rows(w.Lq, seed=7))  # all 360 heads
    print("30 layers", st)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_scoring_normalised_with_the_chunk(cuda_device, dtype):
    """FKV_FLAG_SCORE_WITH_CHUNK: each scoring row's softmax also runs over the
    chunk's own keys (ragged tiles everywhere: T = 200, Lq = 400)."""
    w = wl.scaled(wl.get("480p"), name=f"chunknorm_{dtype}", H=4, T=200, F=7, Fc=2, n_static=2,
                  static_frames=(0, 3, 6), k_dynamic=4, score_stride=3, dtype=dtype, seed=23,
                  score_with_chunk=True)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    st = parity.check_step(w, x, res)
    assert st["score_rel"] <= parity.SCORE_REL


def test_480p_scoring_normalised_with_the_chunk(cuda_device):
    w = wl.scaled(wl.get("480p"), score_with_chunk=True)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    rows = wl.tile_rows(w.Lq, seed=8)
    heads = [(0, h) for h in range(w.H) if x["head_role"][0, h]]
    st = parity.check_step(w, x, res, rows=rows, heads=heads)
    print("480p score_with_chunk", st)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_static_token_masks(cuda_device, dtype):
    """FKV_FLAG_STATIC_TOKEN_MASK: static heads keep fixed token positions; all
    kept lists are token ids; the step, and the cache advance, run on tokens."""
    w = wl.scaled(wl.get("480p"), name=f"tokmask_{dtype}", H=4, T=200, F=7, Fc=2, n_static=2,
                  k_dynamic=3, score_stride=3, dtype=dtype, seed=24, static_token_mask=True)
    x = wl.generate(w)
    assert x["static_mask"].shape == (1, 4, 7 * 200)
    res = parity.run_step(w, x)
    parity.check_step(w, x, res)
    for h in range(w.H):
        if not x["head_role"][0, h]:
            got = parity.gpu_kept(res, 0, h)
            assert got.tolist() == np.flatnonzero(x["static_mask"][0, h].numpy()).tolist()


def test_480p_static_token_masks(cuda_device):
    w = wl.scaled(wl.get("480p"), static_token_mask=True)
    x = wl.generate(w)
    res = parity.run_step(w, x)
    rows = wl.tile_rows(w.Lq, seed=9)
    st = parity.check_step(w, x, res, rows=rows)
    print("480p static token masks", st, res["kept_cnt"].tolist())
