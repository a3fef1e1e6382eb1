"""The multi-GPU path of the benchmark is replicas (the chunk step has no
exchange): each rank runs its own independent step and the job time is the
slowest rank's.  Its host logic runs here as two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import fkv_workloads as wl


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = bench.replica_workload(wl.scaled(wl.get("480p"), T=8, name="mr"), rank, world)
        x = wl.generate(w)
        # ranks draw different inputs but the same shapes
        digest = torch.tensor([float(x["k_hist"].float().sum()), float(x["k_hist"].numel())])
        gathered = [torch.zeros(2) for _ in range(world)]
        dist.all_gather(gathered, digest)
        slow = bench.max_over_ranks(10.0 + rank, dist)
        out[rank] = (gathered[0].tolist(), gathered[1].tolist(), slow,
                     bench.aggregate_throughput(4, world, slow))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_independent_replicas():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    g0, g1, slow, value = out[0]
    assert g0[1] == g1[1]            # same shapes
    assert g0[0] != g1[0]            # different inputs
    assert slow == 11.0 and out[1][2] == 11.0     # max over ranks, seen by every rank
    assert value == pytest.approx(4 * 2 / 0.011)  # all ranks' units / slowest time


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5) == 3.5
    w = wl.get("tiny")
    assert bench.replica_workload(w, 0, 1) is w
    assert bench.replica_workload(w, 1, 2).seed != w.seed
