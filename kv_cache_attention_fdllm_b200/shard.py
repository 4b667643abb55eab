"""Sequence sharding across ranks for the multi-GPU benchmark.

Batch rows of the fused step are independent: each rank owns its own
sequences (caches, index sets, hidden rows) and no data crosses ranks.  The
only collective is the max over ranks of a timing.
"""
from __future__ import annotations

import torch


def rank_sequences(B_per_rank: int, rank: int) -> list:
    """Global sequence ids owned by `rank` when every rank runs B_per_rank sequences."""
    return list(range(rank * B_per_rank, (rank + 1) * B_per_rank))


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank value over the default process group (identity without one)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())
