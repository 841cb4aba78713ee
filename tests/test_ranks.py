"""The multi-rank bookkeeping of bench.py on CPU: two gloo ranks.

Under torchrun every rank times its own copy of the workload (weak scaling,
no data-path collective); the reported time is the slowest rank's and the
reported work the sum over ranks.  These tests run that reduction and the
timing barrier on two CPU processes.
"""
import os
import socket
import sys

import pytest

torch = pytest.importorskip("torch")
import torch.multiprocessing as mp  # noqa: E402

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    r, w, local = bench.dist_env()
    assert (r, w, local) == (rank, world, rank)
    dist = bench.init_group(w, "gloo")
    try:
        bench.barrier(dist)
        # rank r took (r + 1) * 1.5 ms for (r + 1) * 10 units
        t, units = bench.reduce_max_sum(dist, (rank + 1) * 1.5, (rank + 1) * 10.0)
        bench.barrier(dist)
        results[rank] = (t, units)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_to_slowest_time_and_total_work():
    world = 2
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, _free_port(), results), nprocs=world, join=True)
        got = dict(results)
    assert got == {0: (3.0, 30.0), 1: (3.0, 30.0)}


def test_single_rank_needs_no_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.init_group(1, "gloo") is None
    assert bench.reduce_max_sum(None, 2.5, 7.0) == (2.5, 7.0)
    bench.barrier(None)
