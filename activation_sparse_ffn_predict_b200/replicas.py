"""Data-parallel replicas of the decode path: one process per GPU.

The sparse FFN has no cross-GPU exchange: each rank keeps its own copy of the
layer stack and decodes its own token stream, so ranks share no data-path
collective.  The only collectives are for measurement -- a barrier around the
timed region and the maximum of the ranks' elapsed times -- and they work on
any torch.distributed backend (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local: int

    @staticmethod
    def from_env() -> "RankInfo":
        return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                        int(os.environ.get("LOCAL_RANK", "0")))


def token_slice(rank: int, world: int, per_rank: int) -> slice:
    """Positions of this rank's tokens in the seeded stream of world * per_rank tokens."""
    if not (0 <= rank < world) or per_rank < 0:
        raise ValueError("need 0 <= rank < world and per_rank >= 0")
    return slice(rank * per_rank, (rank + 1) * per_rank)


def barrier() -> None:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """The largest value any rank holds (each rank's own value without a group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    dev = device if device is not None else (
        torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu"))
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return units_per_rank * world / (max_ms / 1e3)
