"""Head-sharded execution of the chunk step over several GPUs (one process per
GPU, ``torch.distributed`` for the plumbing).

Every (layer, head) goes through the five steps on its own -- the static
gather, the segment scores, the top-k, the compaction and the attention read
and write only that head's rows (Forcing-KV, ai-feeds.com/i/paper/2605.09681,
"关键模块" 2 and 3 work per head) -- so the L*H heads of a step split into
contiguous ranges, one per rank, with no exchange inside the step.  A rank
runs its range as a step of L' = 1 layer and H' = its head count.  Only a
caller that needs the whole output on every rank pays one collective: an
all-gather of O ([L*H][Lq][D]; NCCL on GPUs, gloo for CPU tests).
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

# Tensors of a step's inputs whose leading two dims are (layer, head).
PER_HEAD_KEYS = ("q_cur", "k_cur", "v_cur", "k_hist", "v_hist", "q_score", "head_role",
                 "static_mask", "k_per_head")


def head_range(num_heads_total: int, world: int, rank: int) -> Tuple[int, int]:
    """[start, stop) of the flattened (layer, head) indices owned by rank:
    contiguous, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    return num_heads_total * rank // world, num_heads_total * (rank + 1) // world


def shard_inputs(x: Dict[str, torch.Tensor], start: int, stop: int) -> Dict[str, torch.Tensor]:
    """The rank's slice of a step's inputs, as one layer of stop - start heads
    (contiguous copies, so the slices can be handed to the C ABI)."""
    out = {}
    for k, t in x.items():
        if k in PER_HEAD_KEYS:
            flat = t.reshape((t.shape[0] * t.shape[1],) + tuple(t.shape[2:]))
            out[k] = flat[start:stop].unsqueeze(0).contiguous()
        else:
            out[k] = t
    return out


def gather_heads(local: torch.Tensor, num_heads_total: int, world: int, group=None) -> torch.Tensor:
    """All-gather per-head results ([1][n_local][...] on each rank, ranges from
    head_range) into [num_heads_total][...] on every rank.  Ranges may differ
    in size by one, so each rank sends a buffer padded to the largest range."""
    import torch.distributed as dist

    flat = local.reshape((-1,) + tuple(local.shape[2:]))
    biggest = max(stop - start for start, stop in
                  (head_range(num_heads_total, world, r) for r in range(world)))
    send = torch.zeros((biggest,) + tuple(flat.shape[1:]), dtype=flat.dtype, device=flat.device)
    send[:flat.shape[0]] = flat
    recv = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(recv, send, group=group)
    parts = []
    for r in range(world):
        start, stop = head_range(num_heads_total, world, r)
        parts.append(recv[r][:stop - start])
    return torch.cat(parts, dim=0)


def local_workload(w, start: int, stop: int, name: Optional[str] = None):
    """The rank's workload description: one layer of stop - start heads of w
    (sizes of every head unchanged)."""
    import dataclasses

    return dataclasses.replace(w, name=name or f"{w.name}[heads {start}:{stop}]", L=1,
                               H=stop - start, layer_seeds=None)
