"""Multi-replica host logic of bench.py on CPU: two gloo ranks (127.0.0.1), each with its
own timed region; the job rate counts every rank's units over the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, units, out):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rate, max_ms = bench.replica_throughput(local_ms[rank], units, world, "cpu")
        out[rank] = (rate, max_ms)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_replicas_use_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    local_ms = [100.0, 150.0]
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, local_ms, 200, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    for r in range(2):
        rate, max_ms = out[r]
        assert max_ms == 150.0                      # max over ranks, seen by every rank
        assert rate == pytest.approx(2 * 200 / 0.150)


def test_single_replica_is_local_time():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    rate, max_ms = bench.replica_throughput(250.0, 100, 1, "cpu")
    assert max_ms == 250.0 and rate == pytest.approx(400.0)
