"""Data-parallel replicas of the BASE layer's hot path: one process per GPU,
each with its own batch of T tokens.

"BASE Layers: Simplifying Training of Large, Sparse Models", Method
(Sharding): every worker solves the balanced assignment of its own tokens, so
the routing needs no exchange between workers; with every expert on every GPU
the forward has no collective at all.  These helpers are the host side of that
arrangement (rank bookkeeping, per-rank inputs, the job's step time as the
max over ranks, whole-job throughput); they run under any process-group
backend (NCCL on GPUs, gloo on CPUs)."""
from __future__ import annotations

import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist

__all__ = ["rank_env", "rank_seed", "max_over_ranks", "job_tokens_per_s"]


def rank_env() -> Tuple[int, int, int]:
    """(rank, world size, local rank) from the launcher's environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int, base: int = 0) -> int:
    """Seed of a rank's own batch: every replica routes different tokens."""
    return base + rank


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The largest value over all ranks (a step's time is its slowest rank's);
    the value itself without a process group or with one rank."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the (max-over-ranks) step time."""
    return tokens_per_rank * world / (ms / 1e3)
