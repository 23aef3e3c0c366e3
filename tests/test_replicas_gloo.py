"""The multi-GPU path of bench.py is replicas only (tokens are independent,
weights replicated, no exchange step). Its host-side aggregation -- the
slowest rank's time and the whole-job token rate -- runs here on two gloo
ranks on the CPU."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 2.0 + rank  # rank 1 is the slower replica
        q.put((rank,) + bench.replica_throughput(1000, local_ms, world, device="cpu"))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, rate, ms in got:
        assert ms == pytest.approx(3.0)
        assert rate == pytest.approx(2 * 1000 / 3e-3)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    rate, ms = bench.replica_throughput(500, 4.0, 1)
    assert ms == 4.0 and rate == pytest.approx(500 / 4e-3)
