"""Multi-rank plumbing for replicas: one process per GPU, no data-path collective.

The path's work units -- (sequence, KV head) -- are independent, so under
torchrun each rank runs its own replica of a workload on its own GPU.  The
only cross-rank traffic is the timing reduction (one float, max over ranks)
and barriers around the timed region.
"""
from __future__ import annotations

import os
from typing import Tuple

import torch
import torch.distributed as dist


def rank_env() -> Tuple[int, int, int]:
    """(rank, world size, local rank) from the torchrun environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_workload(w, rank: int):
    """Rank r's replica draws its own inputs: the workload id of every seed
    tuple is offset by 1000 * r (rank 0 keeps the reference seeds)."""
    return w if rank == 0 else w.scaled(wid=w.wid + 1000 * rank)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a float over all ranks (the identity with one process)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device_sync: bool = True) -> None:
    """Device sync, barrier over ranks, device sync."""
    if device_sync and torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
    if device_sync and torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Aggregate throughput: all ranks' units over the slowest rank's time."""
    return units_per_rank * world / seconds_max
