"""Process-group plumbing for running independent layer replicas, one per GPU.

The layer has no exchange step on one node in this build: each rank runs its
own full copy on its own GPU (weak scaling, no data-path collective). The
process group is used only for barriers around the timed region and for the
max-over-ranks reduction of the measured time.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

import torch
import torch.distributed as dist

__all__ = ["RankInfo", "init_from_env", "barrier", "max_over_ranks", "sum_over_ranks",
           "shutdown"]


@dataclass
class RankInfo:
    rank: int
    world_size: int
    local_rank: int
    initialized: bool


def init_from_env(backend: str = "nccl", timeout_s: int = 120) -> RankInfo:
    """Read RANK / WORLD_SIZE / LOCAL_RANK (torchrun's variables) and, when more
    than one rank is present, join the process group with a short timeout."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return RankInfo(rank, world, local, dist.is_initialized())


def barrier(info: RankInfo) -> None:
    if info.initialized:
        dist.barrier()


def _reduce(value: float, op, info: RankInfo, device) -> float:
    if not info.initialized:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(value: float, info: RankInfo, device="cpu") -> float:
    return _reduce(value, dist.ReduceOp.MAX, info, device)


def sum_over_ranks(value: float, info: RankInfo, device="cpu") -> float:
    return _reduce(value, dist.ReduceOp.SUM, info, device)


def shutdown(info: RankInfo) -> None:
    if info.initialized and dist.is_initialized():
        dist.destroy_process_group()
