"""The multi-rank plumbing of bench.py on CPU with two gloo ranks: one
process per GPU runs independent replicas (no data-path collective), the
ranks meet at barriers around the timed region, the duration is the max over
ranks, and the whole-job rate counts every rank's work.  The reference arm
runs on rank 0 only."""

import io
import os
import socket
import contextlib

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    barrier, allmax, dist = bench.make_comm(world, torch.device("cpu"), "gloo")
    try:
        barrier()
        ms = 10.0 + 5.0 * rank                 # rank 1 is the slow one
        m = allmax(ms)
        barrier()
        rate = bench.whole_job_rate(world, 1e9, m)
        out.put((rank, m, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_whole_job_rate():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == 15.0                                   # the slowest rank's time, on every rank
        assert rate == pytest.approx(2 * 1e9 / 15e-3)      # both ranks' units over that time


def test_single_rank_needs_no_process_group():
    barrier, allmax, dist = bench.make_comm(1, torch.device("cpu"))
    assert dist is None
    barrier()
    assert allmax(3.5) == 3.5
    assert bench.whole_job_rate(1, 2e9, 4.0) == pytest.approx(5e11)


def test_reference_arm_runs_on_rank_zero_only():
    class Args:
        steps, warmup = 1, 3
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Args(), rank=1, world=2)
    assert buf.getvalue() == ""
