"""Process-group plumbing for running the Ring Self-Attention hot path on several GPUs.

Each (batch, head) unit of the method is independent, so N processes (one per GPU) each run
their own batch: there is no collective on the data path. The only cross-rank steps are the
barriers around a timed region and the reduction of the per-rank times (the slowest rank
sets the job's time).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_ranks() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults: one process)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def init(backend: str, timeout_s: float = 120.0, device: torch.device | None = None) -> bool:
    """Join the process group when launched with more than one rank. Returns True if joined."""
    _, world, _ = env_ranks()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    kw = {"backend": backend, "timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(**kw)
    return True


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device: torch.device | None = None) -> float:
    """Maximum of a per-rank scalar over all ranks (identity on one rank)."""
    if not dist.is_initialized():
        return float(x)
    dev = device if device is not None else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(units_per_rank: float, world: int, slowest_seconds: float) -> float:
    """Whole-job throughput when every rank processes `units_per_rank` in its own time and the
    job ends with the slowest rank."""
    if slowest_seconds <= 0:
        raise ValueError("time must be positive")
    return units_per_rank * world / slowest_seconds


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous share of `n_units` for `rank` (sizes differ by at most one)."""
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def finish() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
