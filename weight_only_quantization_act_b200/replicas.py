"""Host logic of multi-GPU runs: independent replicas, one layer per rank.

The AWQ search of one layer runs on one GPU; the layers of a model are independent problems, so N GPUs
run N replicas with no data exchange. The only collective is the timing reduction (max over ranks) that
makes a whole-job throughput out of per-rank device times.
"""
from __future__ import annotations

import dataclasses
import os

from .inputs import Workload


def rank_env():
    """(rank, world_size, local_rank) from the torchrun environment (defaults: a single process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_workload(wl: Workload, rank: int) -> Workload:
    """The layer of rank r: same shapes, its own draw (rank 0 keeps the workload's own seed)."""
    return wl if rank == 0 else dataclasses.replace(wl, number=wl.number + 1000 * rank)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity without an initialised process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank * world / slowest_seconds
