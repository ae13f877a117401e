"""Multi-rank host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

The verify step does not shard (each GPU runs its own replica and verifies
its own tree), so the only cross-rank steps are the barrier around the timed
region and the max over ranks of the device time; both are checked here with
world_size 2, including a rank that arrives late.
"""
import os
import socket
import sys
import time

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        if rank == 1:
            time.sleep(0.5)                       # late rank: the barrier must hold rank 0 back
        t0 = time.perf_counter()
        bench.barrier(world)
        waited = time.perf_counter() - t0
        local = 1.25 + rank                        # per-rank "device seconds"
        m = bench.max_over_ranks(local, world)
        out[rank] = (m, waited)
    finally:
        dist.destroy_process_group()


def test_barrier_and_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == pytest.approx(2.25) and out[1][0] == pytest.approx(2.25)
    assert out[0][1] >= 0.3                     # rank 0 waited for the late rank


def test_single_rank_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert not dist.is_initialized()
