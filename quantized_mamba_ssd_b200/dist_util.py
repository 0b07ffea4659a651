"""Host-side helpers of the multi-GPU benchmark path (one process per GPU).

The prefill shards by batch: each rank scans its own sequences (its own seed), and the only
collective is the max over ranks of the per-rank device times.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_seed(base: int, rank: int) -> int:
    """Seed of a rank's own synthetic batch (rank 0 keeps the workload's seed)."""
    return base + 97 * rank


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank scalar over the process group (the value itself without one)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max * 1e-3)
