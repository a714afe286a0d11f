"""Host-side helpers for running the decode step as replicas on several GPUs.

The (sequence, kv head) units of paged decode attention are independent, so
ranks share nothing on the data path: each rank owns a batch of the
workload's shape and its own block pool.  The only collectives are a barrier
around the timed region and a MAX reduction of the per-rank device times.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s batch: distinct data per replica, same shapes."""
    return base_seed + 7919 * rank


def max_over_ranks(value: float, device=None) -> float:
    """MAX all-reduce of one float (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(bytes_per_rank_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Aggregate GB/s of all ranks over the slowest rank's time."""
    if max_ms <= 0:
        raise ValueError("elapsed time must be positive")
    return bytes_per_rank_per_step * steps * world / (max_ms / 1e3) / 1e9
