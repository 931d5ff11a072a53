"""Rank plumbing for multi-GPU runs (one process per GPU, torch.distributed).

The fusion forward shards with no exchange: examples are independent, so each rank runs the
whole stack on its own examples with replicated weights, and nothing crosses ranks on the data
path. Two ways to give ranks their examples: a fresh batch per rank (weak scaling, as the
benchmark runs), or one batch split into contiguous example ranges balanced by history rows
(shard_batch). A serving request, one history shared by many candidates, splits along its
candidates instead, the history replicated (shard_candidates). The only collective is the timing
reduction (max over ranks).
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


def balanced_ranges(lengths, world: int) -> list:
    """Split one batch's examples into `world` contiguous ranges [b0, b1), balanced by history rows.

    The rows each rank streams through the history-side kernels are its sum of L_b, so the cut
    after rank k's range is put at the example boundary whose prefix sum of lengths lies closest to
    (k + 1) / world of the total. Ranges are contiguous, so a rank's history rows are one slice of
    the layer slab and its offsets only shift. A rank may get no examples (more ranks than examples)."""
    import numpy as np
    L = np.asarray(lengths, dtype=np.int64)
    B = len(L)
    pre = np.concatenate([[0], np.cumsum(L)])
    total = int(pre[-1])
    cuts = [0]
    for k in range(1, world):
        target = total * k / world
        b = int(np.searchsorted(pre, target))        # first boundary with prefix >= target
        if b > 0 and abs(pre[b - 1] - target) <= abs(pre[min(b, B)] - target):
            b -= 1
        cuts.append(min(max(b, cuts[-1]), B))
    cuts.append(B)
    return [(cuts[k], cuts[k + 1]) for k in range(world)]


def shard_batch(tokens, states, offsets, rank: int, world: int):
    """Rank `rank`'s part of one batch: (tokens [b1-b0, N, d], states [n_layers, rows, d],
    offsets rebased to start at 0 (int32 [b1-b0+1]), (b0, b1)). Works on numpy arrays and torch
    tensors alike (slices of the inputs; the offsets are a new array)."""
    import numpy as np
    off = np.asarray(offsets.cpu() if hasattr(offsets, "cpu") else offsets, dtype=np.int64)
    b0, b1 = balanced_ranges(np.diff(off), world)[rank]
    o0, o1 = int(off[b0]), int(off[b1])
    return tokens[b0:b1], states[:, o0:o1], (off[b0:b1 + 1] - o0).astype(np.int32), (b0, b1)


def candidate_range(n_candidates: int, rank: int, world: int) -> tuple:
    """Rank `rank`'s contiguous range [c0, c1) of one request's candidates, as even as whole
    candidates allow (the first n_candidates % world ranks take one more)."""
    base, extra = divmod(max(int(n_candidates), 0), world)
    c0 = rank * base + min(rank, extra)
    return c0, c0 + base + (1 if rank < extra else 0)


def shard_candidates(tokens, tokens_per_candidate: int, rank: int, world: int):
    """Rank `rank`'s part of a serving request whose one history is shared by every candidate.

    Each query token attends over the request's whole history, and the Fusion MLP and the FFN act
    on each token alone, so the request splits along its queries with no exchange: every rank keeps
    the history (and the weights) whole and runs its own candidates' tokens, with n_tokens set to
    that count in its config. tokens: [1, n_candidates * tokens_per_candidate, d] (numpy or torch).
    Returns (tokens [1, (c1-c0) * tokens_per_candidate, d], (c0, c1)); the ranks' outputs, put back
    in rank order along the token axis, are the request's output."""
    n = int(tokens.shape[1])
    if tokens_per_candidate < 1 or n % tokens_per_candidate:
        raise ValueError(f"{n} tokens are not whole candidates of {tokens_per_candidate}")
    c0, c1 = candidate_range(n // tokens_per_candidate, rank, world)
    return tokens[:, c0 * tokens_per_candidate:c1 * tokens_per_candidate], (c0, c1)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar (device time) across ranks; identity for one process."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
