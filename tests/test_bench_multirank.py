"""bench.py's multi-rank reduction on two gloo ranks (CPU, no GPU).

With N GPUs the benchmark runs N independent replicas (the layer has no
exchange step worth sharding at decode sizes); the timed value is the
slowest rank's time and the reported rate counts the units of all ranks.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench

    local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
    slowest = bench.max_over_ranks(local_ms, world)
    rate = bench.whole_job_rate(units_per_rank=1000, world=world, elapsed_ms=slowest)
    out[rank] = (slowest, rate)
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_whole_job_rate():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    assert out[0][0] == pytest.approx(15.0) and out[1][0] == pytest.approx(15.0)
    # 2 ranks x 1000 units in 15 ms
    assert out[0][1] == pytest.approx(2000 / 0.015)
    assert out[1][1] == out[0][1]


def test_single_rank_is_identity():
    import bench

    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_rate(100, 1, 1000.0) == pytest.approx(100.0)
