"""Host-side logic of bench.py, without a GPU.

The multi-rank plumbing (the barrier, the maximum over ranks and the whole-job throughput built on
it) runs as two gloo ranks on this machine.  The ranks are processes started with `spawn` and
rendezvous on 127.0.0.1.  Also checked: under torchrun only rank 0 runs the reference arm (the CPU
oracle) and prints it.
"""
import argparse
import datetime
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_by_rank, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(ms_by_rank[rank], world)
        v, ms = bench.job_throughput(1000.0, ms_by_rank[rank], world)
        out.put((rank, m, v, ms))
        bench.barrier(world)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank():
    """Each rank times its own replica; the job's step is the slowest rank's, and the job's throughput
    counts the units of all ranks over that step."""
    world, ms_by_rank = 2, [2.0, 5.0]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms_by_rank, q)) for r in range(world)]
    for p in procs:
        p.start()
    try:
        res = sorted(q.get(timeout=120) for _ in range(world))
    finally:
        for p in procs:
            p.join(timeout=60)
    assert [p.exitcode for p in procs] == [0, 0]
    assert [r[0] for r in res] == [0, 1]
    for _, m, v, ms in res:
        assert m == 5.0 and ms == 5.0
        assert v == pytest.approx(world * 1000.0 / 5e-3)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.0, 1) == 3.0
    v, ms = bench.job_throughput(10.0, 2.0, 1)
    assert ms == 2.0 and v == pytest.approx(5000.0)


def test_reference_arm_runs_on_rank_zero_only():
    """The other ranks of a torchrun launch leave at once, with no oracle work and nothing printed."""
    args = argparse.Namespace(workload="qwen7b_4k", warmup=3, steps=1, cpu_rows=8)
    assert bench.run_reference(args, rank=1, world=2) is None
