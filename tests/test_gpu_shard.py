"""The head split of the chunk step, run through the CUDA path on one GPU.

Every (layer, head) goes through scoring, selection, compaction and attention
on its own (Forcing-KV, ai-feeds.com/i/paper/2605.09681, "关键模块" 2 and 3
decide per head; Deep Forcing, bxzpzcl.cn/news/2125000, section 3.2 item 2:
each layer compresses its own cache), so a rank that runs its contiguous range
of the flattened (layer, head) indices as a step of its own must produce
exactly the whole step's slices.  Here the ranks' shares run one after another
through ``fkv_step`` on the one GPU (no rank waits for another), and their
outputs, gathered in rank order, are compared bit for bit with one whole-step
call: kept lists, segment scores, compressed K/V and attention output.
"""
import pytest
import torch

import fkv_workloads as wl
import kv_cache_compression_fkv_b200 as fkv
from kv_cache_compression_fkv_b200 import shard
from tests import parity

pytestmark = pytest.mark.gpu

OUTPUTS = ("seg_score", "kept_idx", "kept_cnt", "k_comp", "v_comp", "out")


def _run(w, x_cpu):
    p = fkv.params_for(w)
    o = fkv.allocate(p)
    fkv.step(p, parity.upload(x_cpu), o)
    st = fkv.read_status(o["ws"])
    assert st[0] == 0, st
    return {k: o[k] for k in OUTPUTS}


def _flat(t):
    return t.reshape((t.shape[0] * t.shape[1],) + tuple(t.shape[2:]))


@pytest.mark.parametrize("name,world", [("480p", 3), ("480p", 5), ("480p_3layer", 5),
                                        ("token_small", 4)])
def test_head_shards_equal_the_whole_step(cuda_device, name, world):
    if name == "480p":
        w = wl.get("480p")
    elif name == "480p_3layer":  # ranges that straddle layer boundaries
        w = wl.scaled(wl.get("480p"), name=name, L=3, layer_seeds=(1000, 1001, 1002))
    else:
        w = wl.scaled(wl.get("token14b"), name=name, H=6, T=96, F=9, Fc=2, n_score_q=96,
                      sink_tokens=192, recent_tokens=192, keep_tokens=300, seed=43)
    x = wl.generate(w)
    whole = _run(w, x)
    LH = w.L * w.H
    got = {k: [] for k in OUTPUTS}
    for rank in range(world):
        start, stop = shard.head_range(LH, world, rank)
        part = _run(shard.local_workload(w, start, stop), shard.shard_inputs(x, start, stop))
        for k in OUTPUTS:
            got[k].append(_flat(part[k]))
    for k in OUTPUTS:
        cat = torch.cat(got[k])
        ref = _flat(whole[k])
        if k in ("k_comp", "v_comp"):  # rows past a head's kept count are never written
            rows = (whole["kept_cnt"].reshape(-1) * (w.T if w.granularity == "frame" else 1)).tolist()
            for i, r in enumerate(rows):
                assert torch.equal(cat[i, :r], ref[i, :r]), (k, i)
        elif k == "kept_idx":
            for i, c in enumerate(whole["kept_cnt"].reshape(-1).tolist()):
                assert torch.equal(cat[i, :c], ref[i, :c]), (k, i)
        else:
            assert torch.equal(cat.view(torch.uint8) if cat.is_floating_point() else cat,
                               ref.view(torch.uint8) if ref.is_floating_point() else ref), k
