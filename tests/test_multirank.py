"""The multi-GPU bench path runs one replica per rank; its host logic (barrier,
max over ranks, whole-job aggregation) is checked here with two gloo ranks on
the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        # each rank "measured" a different step time; the job takes the slowest
        ms = [0.130, 0.145][rank]
        worst = bench.max_over_ranks(ms, world)
        value = bench.job_throughput(world, 75.16e9, worst)
        q.put((rank, worst, value))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, worst, value in got:
        assert worst == pytest.approx(0.145)
        assert value == pytest.approx(2 * 75.16e9 / 0.145e-3 / 1e12)


def test_single_rank_aggregation_is_the_plain_rate():
    assert bench.max_over_ranks(0.2, 1) == 0.2
    assert bench.job_throughput(1, 1e12, 1000.0) == pytest.approx(1.0)
