"""Rank plumbing for multi-GPU runs (one process per GPU, torch.distributed).

The fusion forward shards with no exchange: examples are independent, so each rank runs the
whole stack on its own batch (weak scaling) with replicated weights, and nothing crosses ranks
on the data path. The only collective is the timing reduction (max over ranks).
"""
from __future__ import annotations

import os

from . import inputs as I


def rank_env() -> tuple:
    """(rank, world_size, local_rank) from the torchrun environment (defaults: single process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def shard_workload(w: I.Workload, rank: int, world: int) -> I.Workload:
    """Rank `rank`'s batch: the same shapes and distributions, its own examples.

    Weights are drawn from the workload's seed on every rank (replicated); lengths, tokens and
    states from a per-rank seed, so the ranks hold disjoint, independent examples. Rank 0 keeps
    the workload's own seed, so a 1-GPU run and rank 0 of an N-GPU run process the same batch.
    """
    if world <= 1 or rank == 0:
        return w
    return w.replace(seed=w.seed + 1000 * rank, weight_seed=w.weight_seed if w.weight_seed is not None else w.seed)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (device time) across ranks; identity for one process."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
