"""Placement of decode work over ranks (one process per GPU).

Batch sharding: sequences of a decode batch are independent (each reads only
its own cache pages), so a batch shards across GPUs with no exchange on the
data path: a token-balanced assignment of sequences to ranks, and the
max-over-ranks reduction used for timing.

Context parallelism (split-KV across GPUs), for contexts long enough that
one sequence should use several GPUs: every rank holds a contiguous range of
each sequence's pages and decodes it with mla_decode; the partial (u, lse)
of all ranks meet in one all-gather, and mla_merge_partials combines them by
their log-sum-exp on every rank.  This is the one exchange step of the path.
"""
from __future__ import annotations

import heapq
from typing import Callable, Optional, Sequence


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


# ----------------------------------------------------------------------------
# context parallelism
# ----------------------------------------------------------------------------
def split_context(seqlens: Sequence[int], world: int, page_size: int) -> list[list[tuple[int, int]]]:
    """Cut every sequence's cached tokens into `world` contiguous pieces of
    whole pages, one per rank, as even in pages as the count allows (the
    first ranks take one page more).  Returns, per rank, a list over
    sequences of (first_page, n_tokens).  Every piece holds at least one
    token, so each sequence needs at least `world` pages."""
    if world < 1 or page_size < 1:
        raise ValueError("world and page_size must be >= 1")
    out: list[list[tuple[int, int]]] = [[] for _ in range(world)]
    for b, L in enumerate(seqlens):
        L = int(L)
        pages = -(-L // page_size)
        if pages < world:
            raise ValueError(f"sequence {b} has {pages} pages, fewer than {world} ranks")
        base, extra = divmod(pages, world)
        p0 = 0
        for r in range(world):
            n_p = base + (1 if r < extra else 0)
            t0, t1 = p0 * page_size, min(L, (p0 + n_p) * page_size)
            out[r].append((p0, t1 - t0))
            p0 += n_p
    return out


def local_tables(block_table, pieces: Sequence[tuple[int, int]], page_size: int):
    """One rank's block table and sequence lengths for its pieces (numpy,
    int32): row b lists the physical pages of sequence b's piece in order,
    padded with -1; seqlens[b] is the piece's token count."""
    import numpy as np
    bt = np.asarray(block_table)
    n_pages = [-(-n // page_size) for _, n in pieces]
    out = np.full((len(pieces), max(n_pages + [1])), -1, dtype=np.int32)
    for b, ((p0, _), n_p) in enumerate(zip(pieces, n_pages)):
        out[b, :n_p] = bt[b, p0:p0 + n_p]
    return out, np.array([n for _, n in pieces], dtype=np.int32)


def context_parallel_decode(q, kv_cache, block_table, seqlens, page_size: int, d_R: int,
                            softmax_scale: float, group=None,
                            decode_fn: Optional[Callable] = None,
                            merge_fn: Optional[Callable] = None):
    """This rank's part of a context-parallel decode (s_q = 1): decode the
    rank's pieces (block_table / seqlens from local_tables, on this rank's
    device), gather every rank's (u, lse) with one all-gather in rank order,
    and merge them.  Returns (u, lse) of the whole contexts, the same on every
    rank.  decode_fn(q, kv_cache, block_table, seqlens, page_size, d_R,
    softmax_scale) -> (u, lse) and merge_fn(u_parts, lse_parts, u, lse)
    default to the library's decode and mla_merge_partials."""
    import torch
    import torch.distributed as dist
    if q.shape[1] != 1:
        raise ValueError("context parallelism takes one query row per sequence (s_q = 1)")
    if decode_fn is None or merge_fn is None:
        from . import mla
        decode_fn = decode_fn or mla.decode
        merge_fn = merge_fn or mla.mla_merge_partials
    u_loc, lse_loc = decode_fn(q, kv_cache, block_table, seqlens, page_size, d_R, softmax_scale)
    world = dist.get_world_size(group) if (dist.is_available() and dist.is_initialized()) else 1
    # gathered along the leading dimension, rank after rank, then seen as [world, ...]
    B = u_loc.shape[0]
    u_all = torch.empty((world * B,) + tuple(u_loc.shape[1:]), dtype=u_loc.dtype, device=u_loc.device)
    lse_all = torch.empty((world * B,) + tuple(lse_loc.shape[1:]), dtype=lse_loc.dtype,
                          device=lse_loc.device)
    if world > 1:
        dist.all_gather_into_tensor(u_all, u_loc.contiguous(), group=group)
        dist.all_gather_into_tensor(lse_all, lse_loc.contiguous(), group=group)
    else:
        u_all.copy_(u_loc)
        lse_all.copy_(lse_loc)
    u = torch.empty_like(u_loc)
    lse = torch.empty_like(lse_loc)
    merge_fn(u_all.view((world,) + tuple(u_loc.shape)), lse_all.view((world,) + tuple(lse_loc.shape)),
             u, lse)
    return u, lse
