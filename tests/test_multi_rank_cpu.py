"""The N>1 benchmark path on CPU: two gloo ranks, max-over-ranks timing and
the whole-job value (replicas: every rank runs its own step, no data-path
collective)."""

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


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench

    per_rank_ms = [10.0, 12.5][rank]
    m = bench.max_over_ranks(per_rank_ms, world)
    floor = 8.0
    v = bench.step_value(floor, m, world)
    dist.barrier()
    results[rank] = (m, v)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_sum_the_work():
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), results), nprocs=world, join=True)
    for r in range(world):
        m, v = results[r]
        assert m == 12.5                         # slowest rank decides the step time
        assert abs(v - 100.0 * 2 * 8.0 / 12.5) < 1e-9   # both ranks' work counted


def test_single_rank_value():
    import bench

    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert abs(bench.step_value(17.0, 24.0, 1) - 100 * 17 / 24) < 1e-12
