"""Host-side plumbing of the multi-process (one process per GPU) benchmark path.

The hot path shards with no exchange: every (sequence, kv-head) item is independent, so
each rank processes its own sequences and no collective touches the data.  The only
cross-rank steps are the barriers around the timed region and the maximum of the
per-rank times; both go through torch.distributed (NCCL on GPUs, gloo on CPU).
Nothing here computes any part of the method.
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local: int


def rank_info() -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torch.distributed.run (1 process: 0/1/0)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(seed: int, rank: int) -> int:
    """Seed of this rank's synthetic sequences: every rank draws different inputs of the
    same shape (weak scaling: fixed work per rank)."""
    return seed + rank


def barrier(world: int) -> None:
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(world: int, units_per_rank_step: float, steps: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / max_seconds
