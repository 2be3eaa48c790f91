"""Multi-rank host logic of bench.py on CPU processes (gloo, world size 2).

The bench runs one process per GPU, each on its own batch with no collective
on the data path; its only collectives are barriers and one max-reduction of
the timings.  These tests run that reduction and the throughput arithmetic on
two gloo ranks, and check that a rank that dies before the reduction makes the
other rank's collective fail within its timeout instead of waiting forever.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port, timeout_s):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))


def _reduce_worker(rank, world, port, q):
    _init(rank, world, port, 30)
    try:
        # rank r reports times (r + 1) * base: the job takes the slowest rank's time
        mine = [10.0 * (rank + 1), 12.0 * (rank + 1), 1.0 + rank, 5.0 - rank]
        got = bench.max_over_ranks(dist, mine, torch.device("cpu"))
        dist.barrier()
        q.put((rank, got, bench.whole_job_throughput(64, world, 20, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_reduce_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=60) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, value in res:
        assert got == [20.0, 24.0, 2.0, 5.0]                 # element-wise max over ranks
        assert value == pytest.approx(64 * 2 * 20 / 0.020)   # all ranks' tokens / max time


def test_whole_job_throughput_is_weak_scaling_arithmetic():
    assert bench.whole_job_throughput(64, 1, 10, 5.0) == pytest.approx(64 * 10 / 0.005)
    assert bench.whole_job_throughput(64, 4, 10, 5.0) == pytest.approx(
        4 * bench.whole_job_throughput(64, 1, 10, 5.0))


def _dying_worker(rank, world, port, q):
    _init(rank, world, port, 5)
    if rank == 1:
        os._exit(0)          # leaves between steps, without joining the reduction
    try:
        bench.max_over_ranks(dist, [1.0], torch.device("cpu"))
        q.put("returned")
    except Exception as e:   # the surviving rank learns of it through the collective
        q.put(type(e).__name__)


def test_rank_that_exits_makes_the_other_rank_fail_not_hang():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_dying_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    outcome = q.get(timeout=90)
    for p in procs:
        p.join(timeout=90)
    assert outcome != "returned"
