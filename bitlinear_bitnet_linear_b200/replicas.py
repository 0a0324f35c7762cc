"""Data-parallel replicas: host logic for running one independent copy of the
BitLinear workload per GPU (one process per GPU, torch.distributed).

The BitLinear path has no exchange step: each rank owns a full copy of the
packed weights and decodes its own token stream, so no collective touches
the data path.  The process group only carries barriers and the max-over-
ranks reduction of the timed region.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_info():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120, device=None) -> None:
    """Join the process group (no-op for a single process)."""
    _, world, _ = rank_info()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)


def replica_seed(base: int, rank: int) -> int:
    """Seed of a rank's own input stream: distinct per rank, fixed per run."""
    return int(base) + 10_000 * (int(rank) + 1)


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest value over all ranks (the timed region's duration)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return float(units_per_rank) * int(world) / float(seconds_max)
