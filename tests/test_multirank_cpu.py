"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): every rank times its own
batch; the job's time is the max over ranks and its throughput counts every rank's bytes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + rank, 3.0 - rank]       # rank 1 is slower on the first timing, faster on the second
        got = bench.max_over_ranks(local)
        q.put((rank, got))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0] == res[1] == [11.0, 3.0]


def test_max_over_ranks_without_process_group_is_identity():
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]


def test_job_throughput_counts_every_rank():
    one = bench.job_throughput(696_546_432, 1, 0.5)
    assert bench.job_throughput(696_546_432, 8, 0.5) == pytest.approx(8 * one)
    assert one == pytest.approx(696_546_432 / 0.5e-3 / 1e12)
