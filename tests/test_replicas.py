"""The multi-GPU path of bench.py is replicas only: N independent decode
streams, no collective on the data path, the job timed by its slowest
replica. This checks that host logic with two gloo ranks on the CPU."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank: int, world: int, port: int, out):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        ms, rate = bench.replica_rate(10.0 * (rank + 1), 100, world, "cpu")
        out.put((rank, ms, rate))
    finally:
        dist.destroy_process_group()


def test_replica_rate_takes_the_slowest_rank():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, rate in got:
        assert ms == pytest.approx(20.0)            # the slower rank's 20 ms
        assert rate == pytest.approx(2 * 100 / 0.020)  # all ranks' steps over that time


def test_single_replica_needs_no_process_group():
    import bench
    assert bench.replica_rate(5.0, 50, 1) == (5.0, pytest.approx(10000.0))
