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
    mgr = mp.get_context("spawn").Manager()          # no fork of this multi-threaded process
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


def test_reference_arm_under_two_gloo_ranks():
    """`bench.py --impl reference` launched for N > 1 ranks the way a
    multi-GPU run is launched (torch.distributed.run, one node, 127.0.0.1):
    rank 0 alone times the oracle and prints one JSON line; the other rank
    exits 0 without work."""
    import json
    import subprocess
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--impl", "reference", "--steps", "1", "--warmup", "1", "--ctx", "1024", "--layers", "2"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0

