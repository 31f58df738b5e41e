"""Host-side partitioning of the DSA hot path over ranks (one process per GPU).

The path shards by query rows or by sequences:
  - prefill of one sequence: split the query rows into contiguous ranges of equal causal work
    (row t costs t+1 key scores in the indexer and min(k, t+1) gathered keys in attention), each
    rank holding the whole K, V and kI prefix it needs; the ranks' output rows are then
    assembled into the whole sequence on every rank (one broadcast per rank's range: the
    ranges differ in length, so a padded all-gather would move up to twice the bytes);
  - many sequences (prefill batches, decode): whole sequences per rank, no data-path collective.
Timing uses a barrier and the max of the per-rank step times.
"""
from __future__ import annotations

import math


def causal_balanced_row_ranges(L: int, world: int, k: int | None = None, align: int = 1) -> list[tuple[int, int]]:
    """Contiguous query-row ranges [lo, hi) of near-equal work for `world` ranks.

    Work of row t: t+1 (indexer, causal) plus, if k is given, min(k, t+1) (attention); range
    edges are rounded to multiples of `align` (e.g. the indexer's query block).
    """
    if L <= 0 or world <= 0:
        raise ValueError("L and world must be positive")

    def work_upto(n: int) -> float:  # total work of rows [0, n)
        w = n * (n + 1) / 2
        if k is not None:
            m = min(n, k)
            w += m * (m + 1) / 2 + max(0, n - k) * k
        return w

    total = work_upto(L)
    edges = [0]
    for r in range(1, world):
        target = total * r / world
        lo, hi = edges[-1], L
        while lo < hi:  # smallest n with work_upto(n) >= target
            mid = (lo + hi) // 2
            if work_upto(mid) < target:
                lo = mid + 1
            else:
                hi = mid
        e = min(L, max(edges[-1], int(round(lo / align)) * align))
        edges.append(e)
    edges.append(L)
    return [(edges[i], edges[i + 1]) for i in range(world)]


def sequences_for_rank(n_seq: int, world: int, rank: int) -> list[int]:
    """Round-robin assignment of independent sequences to ranks."""
    return list(range(rank, n_seq, world))


def reduce_max(value: float, dist=None, device: str = "cpu") -> float:
    """Max of a per-rank scalar over the process group (identity without one)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: units all ranks processed / the slowest rank's time."""
    if max_seconds <= 0 or not math.isfinite(max_seconds):
        raise ValueError("max_seconds must be positive and finite")
    return units_per_rank * world / max_seconds


def assemble_row_ranges(tensors, ranges: list[tuple[int, int]], dist=None) -> None:
    """Make rows [lo, hi) of every tensor in `tensors` (all indexed by query row along dim 0)
    hold rank r's values for each r's range (lo, hi) = ranges[r], on every rank: rank r
    broadcasts its own rows to the others, in rank order, so every rank issues the same
    collectives in the same order.  Without a process group (or with one rank) nothing moves."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return
    if len(ranges) != dist.get_world_size():
        raise ValueError("one row range per rank")
    for r, (lo, hi) in enumerate(ranges):
        if hi <= lo:
            continue
        for t in tensors:
            dist.broadcast(t[lo:hi], src=r)
