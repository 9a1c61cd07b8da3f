"""The N > 1 bench path on CPU: two gloo ranks (the GPU runs are replicas with
no data-path collective; only the timing reduction crosses ranks)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [120.0, 150.0][rank]          # the ranks' own timed regions
        slowest = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(16 * 1024, 10, world, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_takes_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(2))
    for rank, slowest, value in res:
        assert slowest == 150.0
        assert value == pytest.approx(2 * 16 * 1024 * 10 / 0.150)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_throughput(1024, 4, 1, 1000.0) == pytest.approx(4096.0)
