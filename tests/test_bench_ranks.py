"""The benchmark's multi-GPU mode is replicas only (the decode has no exchange step): every rank
decodes its own copy, the job time is the slowest rank's and the rate counts every rank's bytes.
These run the rank logic as two gloo processes on the CPU."""
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


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        times = [3.0, 5.0]
        slowest = bench.max_over_ranks(times[rank], world, torch.device("cpu"))
        rate = bench.job_rate(1000.0, world, slowest)
        q.put((rank, slowest, rate))
    finally:
        dist.destroy_process_group()


def test_replicas_max_time_and_job_rate():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks see the slowest rank's time; the rate is 2 ranks x 1000 bytes over it
    assert got == [(0, 5.0, 400.0), (1, 5.0, 400.0)]


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(2.5, 1, torch.device("cpu")) == 2.5
    assert bench.job_rate(10.0, 1, 2.0) == pytest.approx(5.0)
