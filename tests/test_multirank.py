"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

With N ranks every rank runs its own replica of the workload (weak scaling,
no collective on the data path), or, for the large-model cache with
``--split heads``, its own slice of every layer's KV heads (strong scaling, no
collective either); the only exchange is the maximum of the per-rank timings,
and the ranks must draw different data.
"""

from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, out):
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        # rank r reports times (r + 1, 10 - r, 0.5 r): the slowest rank decides each entry
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, 0.5 * rank], "cpu", world)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed(rank))
        spans = [None] * world
        dist.all_gather_object(spans, bench.head_split(128, world, rank))
        out.put((rank, got, seeds, spans))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_and_draw_different_data():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, seeds, spans in res:
        assert got == [2.0, 10.0, 0.5]
        assert len(set(seeds)) == world
        assert spans == [(0, 64), (64, 128)]   # the heads of a layer, each exactly once


def test_single_rank_is_identity():
    import importlib

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    assert bench.max_over_ranks([1.5, 2.5], "cpu", 1) == [1.5, 2.5]
    assert bench.rank_seed(0) != bench.rank_seed(1)


def test_head_split_covers_every_head_once():
    import importlib

    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    for world in (1, 2, 4, 8):
        spans = [bench.head_split(128, world, r) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 128
        assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
        assert len({e - b for b, e in spans}) == 1
    with pytest.raises(ValueError):
        bench.head_split(128, 3, 0)
