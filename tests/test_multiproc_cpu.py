"""The N > 1 path of bench.py on CPU: world-size-2 gloo process group, replicas with no
data exchange, timings reduced to the slowest rank, whole-job throughput."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0])
        dist.barrier()
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [2.0, 10.0, 3.0]


def test_job_throughput_is_whole_job():
    import bench
    assert bench.job_throughput(1, 10800, 100, 250.0) == pytest.approx(10800 * 100 / 0.25)
    assert bench.job_throughput(4, 10800, 100, 250.0) == pytest.approx(4 * 10800 * 100 / 0.25)
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
