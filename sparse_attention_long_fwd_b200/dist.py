"""Process-group plumbing for running the NSA forward on several GPUs of one node.

The path partitions into independent problems: each rank runs its own sequences on its
own GPU and nothing crosses ranks on the data path. Ranks only meet to align the timed
region (barrier) and to take the slowest rank's time (max all-reduce)."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def rank_env():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 when absent)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120, device: torch.device | None = None):
    """Initialise the default process group if WORLD_SIZE > 1; returns (world, rank, local)."""
    world, rank, local = rank_env()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if backend == "nccl" and device is not None:
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return world, rank, local


def barrier(world: int):
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """The largest value of x across ranks (every rank must call it)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(total: int, rank: int, world: int):
    """Contiguous split of `total` units (e.g. decode sequences): (start, count) of this rank.
    The first total % world ranks get one extra unit."""
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def aggregate_rate(units_per_rank: int, world: int, max_time_s: float) -> float:
    """Whole-job throughput: all ranks' units divided by the slowest rank's time."""
    return units_per_rank * world / max_time_s
