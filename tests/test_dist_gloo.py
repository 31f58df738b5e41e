"""Multi-rank host logic on CPU with world-size-2 gloo process groups."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from dsa_lightning_indexer_02_b200.sharding import (assemble_row_ranges, causal_balanced_row_ranges, reduce_max,
                                                    sequences_for_rank, weak_scaling_value)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, L, k, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ranges = causal_balanced_row_ranges(L, world, k=k, align=8)
        lo, hi = ranges[rank]
        # each rank "times" its own slice; the job time is the max over ranks
        my_work = sum(t + 1 + min(k, t + 1) for t in range(lo, hi))
        mx = reduce_max(float(my_work), dist)
        seqs = sequences_for_rank(16, world, rank)
        import torch
        got = [None] * world
        dist.all_gather_object(got, (lo, hi, my_work, seqs))
        q.put((rank, mx, got))
    finally:
        dist.destroy_process_group()


def test_two_rank_partition_and_max_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    L, k, world = 20000, 2048, 2
    procs = [ctx.Process(target=_worker, args=(r, world, port, L, k, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, got in res:
        (lo0, hi0, w0, s0), (lo1, hi1, w1, s1) = got
        assert lo0 == 0 and hi0 == lo1 and hi1 == L          # contiguous cover of all rows
        assert hi0 % 8 == 0
        assert mx == max(w0, w1)                             # max over ranks
        assert abs(w0 - w1) / (w0 + w1) < 0.01               # causal work balanced
        assert sorted(s0 + s1) == list(range(16)) and not set(s0) & set(s1)


def test_partition_edge_cases():
    assert causal_balanced_row_ranges(5, 1) == [(0, 5)]
    r = causal_balanced_row_ranges(3, 4)
    assert r[0][0] == 0 and r[-1][1] == 3 and all(a <= b for a, b in r)
    r = causal_balanced_row_ranges(131072, 8, k=2048, align=8)
    works = [sum(t + 1 + min(2048, t + 1) for t in range(lo, hi)) for lo, hi in r]
    assert max(works) / min(works) < 1.01
    # later ranks get fewer rows (rows near the end carry more keys)
    assert (r[0][1] - r[0][0]) > (r[-1][1] - r[-1][0])
    assert weak_scaling_value(131072, 4, 0.2) == 131072 * 4 / 0.2
    with pytest.raises(ValueError):
        weak_scaling_value(1, 1, 0.0)
    assert reduce_max(3.5) == 3.5


def _row_value(t: int, h: int) -> float:
    """Stand-in for one query row's output (what the per-rank prefill call would write)."""
    return float(t * 1000 + h)


def _split_worker(rank, world, port, L, k, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ranges = causal_balanced_row_ranges(L, world, k=k, align=8)
        lo, hi = ranges[rank]
        out = torch.full((L, 3), -1.0)                     # rows outside this rank's range: garbage
        idx = torch.full((L, 4), -7, dtype=torch.int32)
        for t in range(lo, hi):                            # the per-rank call, on its own rows only
            out[t] = torch.tensor([_row_value(t, h) for h in range(3)])
            idx[t] = torch.arange(4, dtype=torch.int32) + t
        assemble_row_ranges((out, idx), ranges, dist)
        q.put((rank, ranges, out.numpy().copy(), idx.numpy().copy()))
    finally:
        dist.destroy_process_group()


def test_two_rank_row_split_assembles_the_whole_sequence():
    """One sequence split by causal-balanced query-row ranges over two gloo ranks: after the
    assembly every rank holds every row, each written by the rank that owns it, in row order."""
    import numpy as np
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    L, k, world = 3000, 256, 2
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, L, k, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_out = np.array([[_row_value(t, h) for h in range(3)] for t in range(L)])
    want_idx = np.arange(L)[:, None] + np.arange(4)[None, :]
    for rank, ranges, out, idx in res:
        (a0, b0), (a1, b1) = ranges
        assert a0 == 0 and b0 == a1 and b1 == L and b0 - a0 > b1 - a1     # uneven row counts
        assert np.array_equal(out, want_out), rank
        assert np.array_equal(idx, want_idx), rank


def test_assembly_without_a_process_group_is_a_no_op():
    import torch
    t = torch.arange(6.0)
    assemble_row_ranges((t,), [(0, 6)], None)
    assert torch.equal(t, torch.arange(6.0))
