"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

Decode shards over (sequence, kv-head) units with no data exchange, so the
only cross-rank steps are the barrier and the max-over-ranks reduction of the
timed duration; `value` is the bytes of all ranks over the slowest rank's
time.
"""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        dist.barrier()
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        slowest = bench.reduce_max(local_ms, dist, torch.device("cpu"))
        value = bench.throughput_gbs(1_000_000_000, world, 4, slowest)
        results[rank] = (slowest, value)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    assert set(results.keys()) == {0, 1}
    for rank in range(world):
        slowest, value = results[rank]
        assert slowest == pytest.approx(15.0)
        # 2 ranks x 4 steps x 1 GB over 15 ms
        assert value == pytest.approx(2 * 4 * 1.0 / 0.015)


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.reduce_max(3.5, None, None) == 3.5
    assert bench.throughput_gbs(580_000_000, 1, 1000, 100.0) == pytest.approx(5800.0)
