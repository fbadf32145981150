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


def _ref_args(**kw):
    a = dict(workload="tiny_f32", warmup=0, steps=1, cpu_rows=16, ref_prefix=256, route="soft", tiers=7, paths=1,
             block_sparse=False)
    a.update(kw)
    return argparse.Namespace(**a)


def test_reference_arm_prints_the_main_arms_config():
    """Both arms describe the workload with the same config object, so the two lines compare."""
    args = _ref_args()
    res = bench.run_reference(args, rank=0, world=1)
    assert res["impl"] == "reference"
    assert res["config"] == bench.workload_config(bench.workload_cfg(args, "tiny_f32"), 1)
    assert res["value"] > 0 and res["ms_per_step"] > 0
    assert "extrapolated" in res["value_is"]


def test_recall_check_counts_a_planted_mismatch():
    """The bench's recall check finds no mismatch for the oracle's own recall, and counts one row
    whose list is reversed (no hash bit of these inputs lies within 1e-4 of zero)."""
    import numpy as np
    import oracle
    from fastmka_inputs import CONFIGS, make_inputs, to_f64
    cfg = CONFIGS["tiny_f32"]
    inp = make_inputs(cfg)
    X = to_f64(inp.x)
    summ = oracle.block_summaries(X, cfg.block)[0]
    idx, *_ = oracle.longterm_recall(X[0], np.arange(cfg.seq), summ, to_f64(inp.hash_proj), cfg.block, cfg.recall_r)
    got = idx[None].copy()
    r = bench.recall_check(cfg, inp, got)
    assert (r["mismatches_unexcused"], r["mismatches_excused"], r["rows_checked"]) == (0, 0, cfg.seq)
    got[0, 200] = got[0, 200][::-1]
    assert bench.recall_check(cfg, inp, got)["mismatches_unexcused"] == 1


def test_hbm_bytes_of_the_headline_workload():
    """The fuse reads the projected sources once and writes K and V once: at 1 x 131072 with
    2 * d_kv = 2048 columns that is at least 1.07 GB + 0.54 GB."""
    from fastmka_inputs import CONFIGS
    b = bench.prefill_hbm_bytes(CONFIGS["llama8b_128k"])
    assert b["route_fuse"] >= 131072 * 2048 * (4 + 2)
    assert b["block_codes"] >= 131072 * 4096 * 2


def test_sustained_peak_only_under_the_power_cap():
    peaks = {"bf16_tflops": 1654.3, "bf16_tflops_sustained": 1391.4, "hbm_gbs": 6457.7, "source": "measured"}
    from fastmka_inputs import CONFIGS
    cfg = CONFIGS["llama8b_128k"]
    capped = {"sm_mhz": 1552.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    full = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    assert bench.power_capped(capped) and not bench.power_capped(full) and not bench.power_capped(None)
    r = bench.attention_roofline(cfg, 140.0, peaks, sustained=True)
    assert r["peak"] == 1391.4 and r["frac_of_burst_peak"] < r["frac"]
    assert bench.attention_roofline(cfg, 140.0, peaks)["peak"] == 1654.3
