"""Rank plumbing for running independent replicas of the attention step, one process
per GPU.  Every context-parallel rank of the method is a virtual rank on one GPU, so
several GPUs run independent replicas: no data-path collective, only a barrier around
the timed region and a max-reduction of the measured time."""
from __future__ import annotations

import dataclasses
import os

import torch
import torch.distributed as dist


@dataclasses.dataclass
class RankInfo:
    rank: int
    world: int
    local_rank: int
    distributed: bool


def init_from_env(backend: str = "nccl", timeout_s: float = 120.0) -> RankInfo:
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        import datetime
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return RankInfo(rank, world, local, world > 1)


def barrier(info: RankInfo) -> None:
    if info.distributed:
        dist.barrier()


def max_over_ranks(info: RankInfo, value: float, device=None) -> float:
    """The largest `value` over all ranks (every rank gets it)."""
    if not info.distributed:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return units_per_rank * world / max_seconds


def finalize(info: RankInfo) -> None:
    if info.distributed and dist.is_initialized():
        dist.destroy_process_group()
