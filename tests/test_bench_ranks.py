"""The multi-rank host logic of bench.py on CPU: two gloo ranks with
different step times agree on the slowest rank's time, and the whole-job
rate counts the units of both ranks over that time (replicas, weak
scaling)."""
import os
import socket
from datetime import timedelta

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, seconds, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        t = bench.max_over_ranks(seconds[rank], world, dist, "cpu")
        r = bench.job_rate(1000.0, seconds[rank], world, dist, "cpu")
        q.put((rank, t, r))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time():
    world, seconds = 2, [0.5, 0.8]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, seconds, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, t, r in got:
        assert t == max(seconds)
        assert r == world * 1000.0 / max(seconds)


def test_single_rank_needs_no_group():
    import bench
    assert bench.max_over_ranks(0.25, 1) == 0.25
    assert bench.job_rate(100.0, 0.25, 1) == 400.0
