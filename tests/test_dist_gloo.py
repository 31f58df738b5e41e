"""Multi-rank host logic on CPU with world-size-2 gloo process groups."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from dsa_lightning_indexer_02_b200.sharding import (causal_balanced_row_ranges, reduce_max, sequences_for_rank,
                                                    weak_scaling_value)


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
