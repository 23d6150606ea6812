"""Data-parallel placement of decode work over ranks (one process per GPU).

Sequences of a decode batch are independent: each one reads only its own
cache pages, so a batch shards across GPUs with no exchange on the data path.
This module holds the host-side pieces of that: a token-balanced assignment
of sequences to ranks, and the max-over-ranks reduction used for timing.
"""
from __future__ import annotations

import heapq
from typing import Sequence


def partition_sequences(seqlens: Sequence[int], world: int) -> list[list[int]]:
    """Assign sequences to `world` ranks, balancing cached tokens.

    Longest-first greedy: each sequence goes to the rank with the fewest
    tokens so far (ties to the lower rank).  Deterministic, so every rank
    computes the same assignment without communicating.  The most loaded
    rank holds at most 4/3 of the optimum (Graham's bound for this rule).
    Each rank's list is in ascending sequence order.
    """
    if world < 1:
        raise ValueError("world must be >= 1")
    order = sorted(range(len(seqlens)), key=lambda b: (-int(seqlens[b]), b))
    heap = [(0, r) for r in range(world)]
    parts: list[list[int]] = [[] for _ in range(world)]
    for b in order:
        load, r = heapq.heappop(heap)
        parts[r].append(b)
        heapq.heappush(heap, (load + int(seqlens[b]), r))
    return [sorted(p) for p in parts]


def rank_load(seqlens: Sequence[int], part: Sequence[int]) -> int:
    return sum(int(seqlens[b]) for b in part)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over the default process group (identity
    when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
