"""The replica (N > 1) bookkeeping of bench.py on CPU: two gloo ranks, each with its own
step time, agree on the max over ranks and on the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(times[rank], dist)
        value = bench.job_tokens_per_s(world, 16384, 10, ms_max)
        results[rank] = (ms_max, value)
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank():
    world, times = 2, [12.5, 20.0]
    results = mp.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), times, results), nprocs=world,
                       start_method="spawn", join=True)
    assert results[0][0] == results[1][0] == 20.0
    assert results[0][1] == pytest.approx(2 * 16384 * 10 / 0.020)
    assert results[0][1] == results[1][1]


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0) == 3.0
    assert bench.job_tokens_per_s(1, 100, 4, 2.0) == pytest.approx(200000.0)
