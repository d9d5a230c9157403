"""Replica-parallel plumbing for several GPUs of one node.

The layer's hot path has no exchange step (prefill sequences and decode
batches are independent), so N ranks run N independent replicas of the
workload on their own GPUs (weak scaling) and only the timing is reduced:
the job's time is the slowest rank's, and its throughput counts the units of
every rank.  Nothing here touches a GPU; the functions take the process
group's device for the single-scalar reduction (a CUDA device under NCCL,
the CPU under gloo).
"""
from __future__ import annotations

import os


def rank_world() -> tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(rank: int, base: int = 0) -> int:
    """Seed of a rank's synthetic inputs: each replica draws its own workload."""
    return base + rank


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank scalar over all ranks (the job time is the
    slowest replica's); the identity when no process group is initialised."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_replica: float, world: int, seconds: float) -> float:
    """Whole-job throughput: every replica's units over the slowest replica's time."""
    if seconds <= 0:
        raise ValueError("job_rate: non-positive time")
    return world * units_per_replica / seconds
