"""CPU tests of the multi-rank benchmark plumbing with the gloo backend (world size 2).

The decode path shards by slot with no exchange step, so N GPUs run N independent
replicas; what needs checking is the rank-side timing rule: every rank takes the same
collective steps, the reported time is the max over ranks, and the rate counts the
units of all ranks."""
import os
import socket

import pytest
import torch
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        my_ms = [12.5, 20.0][rank]
        worst = bench.max_over_ranks(my_ms, dist)
        dist.barrier()
        rate = bench.whole_job_rate(1000, world, worst)
        q.put((rank, worst, rate))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, rate in got:
        assert worst == 20.0
        assert rate == pytest.approx(2 * 1000 / 0.020)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.0, None) == 3.0
    assert bench.whole_job_rate(500, 1, 10.0) == pytest.approx(50_000)
