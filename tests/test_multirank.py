"""Host logic of the N > 1 path on CPU: two gloo ranks each time their own independent work, the
job's time is the slowest rank's, and throughput counts every rank's units."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]                        # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world)
        q.put((rank, got, bench.job_throughput(4096, 10, world, got)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in res:
        assert got == 20.0
        assert thr == pytest.approx(4096 * 2 * 10 / 0.020)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25
    assert bench.job_throughput(64, 1000, 1, 50.0) == pytest.approx(64 * 1000 / 0.05)
