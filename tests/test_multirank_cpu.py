"""The benchmark's multi-rank host logic on CPU ranks (gloo, world size 2): the timed
region's elapsed time is the max over ranks, the reported value counts every rank's steps
(weak scaling: one batch per GPU), and the reference arm does its work on rank 0 only.
No GPU is used and no collective runs on a data path."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 20.0][rank]                              # rank 1 is the slow one
        slowest = bench.max_over_ranks(ms, world, "cpu")
        value = bench.aggregate_value(100, world, slowest)
        dist.barrier()
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, slowest, value in got:
        assert slowest == 20.0                               # max, not the local time
        assert value == pytest.approx(2 * 100 / 0.020)       # both ranks' steps / slowest time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1, "cpu") == 3.0
    assert bench.aggregate_value(10, 1, 5.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        pass
    args = A()
    assert bench.run_reference(args, rank=1) is None         # returns at once, prints nothing
    assert capsys.readouterr().out == ""
