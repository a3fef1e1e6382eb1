"""Head-sharded execution (the multi-GPU split of the chunk step): the
partition, the per-rank input slices, and the all-gather of O, as gloo ranks
on the CPU.  The per-head computation is the oracle's, so a sharded step must
reproduce the whole step exactly (every head runs alone in both)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import fkv_workloads as wl
from kv_cache_compression_fkv_b200 import shard
from oracle import fkv_oracle as orc


@pytest.mark.parametrize("LH", [1, 7, 12, 40, 360])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_head_range_partitions_every_head_once(LH, world):
    ranges = [shard.head_range(LH, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == LH
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def _oracle_step(x, w):
    f = {k: wl.as_float64(x[k]) for k in ("q_cur", "k_cur", "v_cur", "k_hist", "v_hist")}
    return orc.step(f["q_cur"], f["k_cur"], f["v_cur"], f["k_hist"], f["v_hist"],
                    x["head_role"].numpy(), x["static_mask"].numpy(), x["k_per_head"].numpy(),
                    T=w.T, granularity=w.granularity, scale=1.0 / np.sqrt(w.D),
                    score_stride=w.score_stride)


def _tiny():
    return wl.scaled(wl.get("tiny"), name="shard_tiny", L=2, layer_seeds=(5, 6))


def test_sharded_oracle_step_equals_whole_step():
    w = _tiny()
    x = wl.generate(w)
    whole = _oracle_step(x, w)
    LH, world = w.L * w.H, 3
    for rank in range(world):
        start, stop = shard.head_range(LH, world, rank)
        xl = shard.shard_inputs(x, start, stop)
        assert xl["k_hist"].shape[:2] == (1, stop - start) and xl["k_hist"].is_contiguous()
        part = _oracle_step(xl, shard.local_workload(w, start, stop))
        for i, g in enumerate(range(start, stop)):
            l, h = divmod(g, w.H)
            assert np.array_equal(part["kept"][(0, i)], whole["kept"][(l, h)])
            assert np.array_equal(part["out"][(0, i)], whole["out"][(l, h)])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # uneven ranges: 7 heads over the ranks
        LH = 7
        start, stop = shard.head_range(LH, world, rank)
        local = torch.stack([torch.full((3, 2), float(g)) + torch.arange(6.0).reshape(3, 2)
                             for g in range(start, stop)]).unsqueeze(0)
        full = shard.gather_heads(local, LH, world)
        want = torch.stack([torch.full((3, 2), float(g)) + torch.arange(6.0).reshape(3, 2)
                            for g in range(LH)])
        ok_synthetic = bool(torch.equal(full, want))
        # the oracle step of this rank's heads, gathered, against the whole step
        w = _tiny()
        x = wl.generate(w)
        s0, s1 = shard.head_range(w.L * w.H, world, rank)
        part = _oracle_step(shard.shard_inputs(x, s0, s1), shard.local_workload(w, s0, s1))
        o_local = torch.from_numpy(np.stack([part["out"][(0, i)] for i in range(s1 - s0)])).unsqueeze(0)
        o_full = shard.gather_heads(o_local, w.L * w.H, world)
        whole = _oracle_step(x, w)
        want_o = np.stack([whole["out"][divmod(g, w.H)] for g in range(w.L * w.H)])
        out[rank] = (ok_synthetic, bool(np.array_equal(o_full.numpy(), want_o)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_the_whole_output(world):
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    for r in range(world):
        assert out[r] == (True, True), (r, out[r])
