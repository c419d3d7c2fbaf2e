"""The benchmark's multi-rank plumbing on CPU: two `gloo` ranks (one process
each) take the maximum of their step times, agree on the whole-job value and
only rank 0 runs the reference arm.  The GPU work itself is per rank and has
no collective, so this is the whole N > 1 path apart from the kernels."""

import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        ms = 2.0 + 1.5 * rank  # rank 1 is the slow one
        worst = bench.max_over_ranks_of(ms, world, torch.device("cpu"))
        value = bench.whole_job_tflops(1e12, worst, world)
        bench.rank_barrier(world)
        out.put((rank, worst, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(out.get(timeout=5) for _ in range(world))
    for rank, worst, value in res:
        assert worst == 3.5
        # 1 TFLOP per rank and step, 2 ranks, 3.5 ms at the slowest rank
        assert value == pytest.approx(2 * 1.0 / 3.5e-3)


def test_single_rank_needs_no_collective():
    assert bench.max_over_ranks_of(4.25, 1, None) == 4.25
    bench.rank_barrier(1)
    assert bench.whole_job_tflops(2e12, 4.0, 1) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class Args:
        steps, warmup = 1, 3
    bench.run_reference(Args(), rank=1, world=2)  # returns at once, prints nothing
    assert capsys.readouterr().out == ""
