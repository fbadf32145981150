#!/usr/bin/env python
"""FastMKA layer benchmark on B200.

Headline: prefill tokens/s of the Llama-3.1-8B-shaped FastMKA layer (batch 1 x
seq 131072, bf16; every step runs the whole layer: projections, router, L2 EMA,
L3 hash recall, route-fuse, causal GQA attention), the largest workload that
fits one GPU.  Alongside it: the same measurement for the smaller prefill
workloads (by_workload), decode us/token over fused caches of 4K-256K positions
(256 steps in one CUDA graph), the roofline fraction of the attention and the
HBM fraction of every bandwidth-bound stage (measured live with CUDA events on
the launching stream), the end-to-end rate through host buffers, the recalled
blocks checked against the CPU oracle, and the CPU oracle's own rate.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

With N > 1 (torchrun, one rank per GPU) every rank runs an independent replica
of the workload (the layer shards by sequence with no exchange): weak scaling.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fastmka_inputs import CONFIGS, make_inputs, sample_rows, to_f64  # noqa: E402

REASON_BITS = {  # nvidia-smi clocks_event_reasons bitmask
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    0x100: "display_clock_setting",
}
PREFILL_STAGES = ["projection_gemm", "router_tail", "token_codes", "block_sums", "block_codes", "ema_carry", "recall",
                  "route_fuse", "attention", "state_tail"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu),
                 "--query-gpu=index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        if not getattr(self, "out", ""):
            return None
        sm, mx, reasons, power = [], [], 0, []
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 5:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
                reasons |= int(f[4], 16)
            except ValueError:
                continue
        if not sm:
            return None
        loaded = [s for s, p in zip(sm, power) if p > 200.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "samples": len(sm),
                "power_w_max": max(power), "reasons": [n for b, n in REASON_BITS.items() if reasons & b]}


# ------------------------------------------------------------------ workload arithmetic
def prefill_flops(cfg) -> dict:
    T, d, dq, dkv, rh, nb = cfg.tokens, cfg.d_model, cfg.dq, cfg.dkv, cfg.router_hidden, cfg.hash_bits
    causal_pairs = cfg.batch * cfg.seq * (cfg.seq + 1) / 2
    attn = 4.0 * cfg.d_head * cfg.n_q_heads * causal_pairs  # QK^T and PV over j <= t only
    if getattr(cfg, "block_sparse", 0):
        # Block-MKA: row t attends to keys <= t of its own block and to min(R, t // b) recalled blocks
        t = np.arange(cfg.seq)
        keys = t % cfg.block + 1 + (np.minimum(cfg.recall_r, t // cfg.block) * cfg.block if cfg.tiers & 4 else 0)
        attn = 4.0 * cfg.d_head * cfg.n_q_heads * cfg.batch * float(keys.sum())
    if getattr(cfg, "attention_paths", 1) == 3 and cfg.tiers & 4:
        # full MKA's recalled-block path: row t attends to min(R, t // b) blocks of b keys
        t = np.arange(cfg.seq)
        keys = np.minimum(cfg.recall_r, t // cfg.block) * cfg.block
        attn += 4.0 * cfg.d_head * cfg.n_q_heads * cfg.batch * float(keys.sum())
    return {"projections": 2.0 * T * d * (dq + 2 * dkv + 2 * rh + nb), "attention": attn}


def decode_bytes_per_token(cfg, ctx: int, ntot: int) -> float:
    w = ntot * cfg.d_model * 2                       # packed projection weights, bf16
    cache = ctx * cfg.dkv * 2 * 2                    # K and V rows read by the attention
    state = 2 * cfg.dkv * 4 * (cfg.recall_r + 4) + cfg.d_model * 8 * 2
    return float(w + cache + state)


def workload_cfg(args, name):
    """The named workload with the routing gate / memory tiers the command line selects (and, for
    profiling runs, another sequence length of the same shape)."""
    c = CONFIGS[name].replace(route_mode=args.route, tiers=args.tiers,
                              attention_paths=getattr(args, "paths", 1),
                              block_sparse=int(getattr(args, "block_sparse", False)))
    seq = getattr(args, "seq", None)
    return c.replace(seq=seq) if seq and name == args.workload else c


def model_name(cfg) -> str:
    return "Llama-3.1-8B" if cfg.name.startswith("llama") else "Qwen2.5-7B"


def prefill_kernels(cfg) -> int:
    """Kernel launches of one prefill call: projection GEMM, router softmax, token codes, block
    sums, block sums of X and block codes (two), EMA carries, recall, fuse, attention."""
    return 10


FFMA_LANES_PER_SM = 128  # fp32 FMA lanes of an sm_100 SM (4 SMSPs x 32)


def ffma_peak_tflops(sm_max_mhz: float = 1965.0, sms: int = 148) -> float:
    """Dense fp32 FFMA peak: SMs x FMA lanes x 2 flops x the maximum SM clock."""
    return sms * FFMA_LANES_PER_SM * 2 * sm_max_mhz * 1e6 / 1e12


def prefill_hbm_bytes(cfg) -> dict:
    """Algorithmic DRAM bytes per prefill call of each bandwidth-bound stage (each input read once,
    each output written once; workspace tensors the GEMM wrote count as reads)."""
    T, d, W, nb, R = cfg.tokens, cfg.d_model, 2 * cfg.dkv, cfg.hash_bits, cfg.recall_r
    elem = 4 if cfg.dtype == "f32" else 2
    nblk = cfg.batch * (cfg.seq // cfg.block)
    rh_parts = max(1, cfg.router_hidden // 128)
    return {
        "router_tail": T * rh_parts * 3 * 4 + T * 3 * 4,
        "token_codes": T * nb * 4 + T * 4,
        "block_sums": T * W * 4 + nblk * 9 * W * 4,
        "block_codes": T * d * elem + nblk * 4,
        "recall": T * 4 + nblk * 4 + T * (R + 1) * 4,
        "route_fuse": T * W * 4 + T * 3 * 4 + T * R * 4 + nblk * W * 4 + T * W * elem,
    }


def workload_config(cfg, world: int) -> dict:
    """The `config` object of the JSON line, the same for both arms."""
    return {"workload": f"{cfg.name}: {model_name(cfg)}-shaped FastMKA layer prefill, batch {cfg.batch} x seq "
                        f"{cfg.seq}, d_model {cfg.d_model}, {cfg.n_q_heads}/{cfg.n_kv_heads} heads, d_h "
                        f"{cfg.d_head}, router {cfg.dq}->{cfg.router_hidden}->3, alpha {cfg.alpha}, L3 block "
                        f"{cfg.block}, R {cfg.recall_r}, nbits {cfg.hash_bits}, {cfg.dtype}, seed {cfg.seed}"
                        + ("" if (cfg.route_mode, cfg.tiers) == ("soft", 7) else
                           f"; routing {cfg.route_mode}, tiers mask {cfg.tiers}")
                        + ("; full MKA, three attention paths" if cfg.attention_paths == 3 else "")
                        + ("; Block-MKA block-sparse attention" if cfg.block_sparse else ""),
            "global_batch": cfg.batch * world, "seq_len": cfg.seq,
            "parallelism": f"replicas x{world} (independent sequences, no exchange)",
            "l2": "flushed (512 MB write) before every timed step"}


def power_capped(clocks) -> bool:
    """Whether the timed region ran in the power-capped regime: sw_power_cap active and the median
    SM clock under load below 95% of the maximum."""
    return bool(clocks) and "sw_power_cap" in clocks.get("reasons", []) and \
        clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"]


def attention_roofline(cfg, attn_ms: float, peaks: dict, clk_max_mhz: float = 1965.0, sustained=False) -> dict:
    fl = prefill_flops(cfg)["attention"]
    tf = fl / (attn_ms / 1e3) / 1e12
    kernel = (("attention (Block-MKA block-sparse: own block + recalled blocks)" if cfg.block_sparse else
               "attention (causal GQA, online max-shift)") if cfg.attention_paths == 1 else
              "attention (full MKA: causal pass + recalled-block pass)")
    if cfg.dtype == "f32":
        peak = ffma_peak_tflops(clk_max_mhz)
        return {"kernel": kernel + ", fp32 FFMA", "bound": "alu", "achieved": round(tf, 2), "peak": round(peak, 1),
                "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                "peak_source": f"derived: 148 SMs x {FFMA_LANES_PER_SM} FP32 lanes x 2 x {clk_max_mhz:.0f} MHz",
                "traffic": None, "avg_ms": round(attn_ms, 4), "flops_per_launch": fl}
    peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    how = ("sustained: the kernel runs for seconds back to back and the timed region's clocks show the "
           "power cap" if sustained else "burst: the kernel is timed alone per step at full clocks")
    return {"kernel": kernel, "bound": "tensor", "achieved": round(tf, 1), "peak": peak,
            "unit": "TFLOP/s", "frac": round(tf / peak, 4),
            "peak_source": f"{peaks['source']} bf16 dense cuBLAS ({how})",
            "frac_of_burst_peak": round(tf / peaks["bf16_tflops"], 4),
            "traffic": traffic_from_profiles("attention_tc", cfg.name), "avg_ms": round(attn_ms, 4),
            "flops_per_launch": fl}


def hbm_rooflines(cfg, stage_ms: dict, peaks: dict) -> dict:
    """GB/s and fraction of the measured HBM copy bandwidth of each bandwidth-bound stage, from its
    algorithmic bytes and its own CUDA-event time (stages run one after another when timed)."""
    out = {}
    for k, b in prefill_hbm_bytes(cfg).items():
        ms = stage_ms.get(k)
        if not ms:
            continue
        gbs = b / (ms / 1e3) / 1e9
        out[k] = {"bytes": int(b), "ms": round(ms, 4), "achieved": round(gbs, 1), "unit": "GB/s",
                  "frac": round(gbs / peaks["hbm_gbs"], 4)}
    return {"peak": peaks["hbm_gbs"], "peak_source": f"{peaks['source']} HBM copy bandwidth", "kernels": out}


def measure_prefill(args, cfg, dev, world, steps, warmup, with_e2e=False, with_clocks=False):
    """Prefill tokens/s of one workload: `warmup` untimed calls, stage times from profiled calls
    (every stage alone on the caller's stream), then `steps` timed calls with L2 flushed before
    each (device time by CUDA events, independent memory kernels as concurrent branches)."""
    import route_kv_memory_b200 as mka
    inp = make_inputs(cfg)
    weights = {k: v.to(dev) for k, v in inp.tensors().items() if k != "x"}
    layer = mka.FastMKALayer(cfg, weights, dev)
    x = inp.x[:, :cfg.seq].contiguous().to(dev)
    out = torch.empty(cfg.batch, cfg.seq, cfg.dq, dtype=x.dtype, device=dev)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()

    for _ in range(warmup):
        layer.prefill(x, out)
    torch.cuda.synchronize()
    assert mka.mka_status() == 0

    stage_ms = []
    mka.mka_profile_enable(True)
    for i in range(min(steps, 10)):
        flush.zero_()
        layer.prefill(x, out)
        stage_ms.append(mka.mka_profile_read())
    mka.mka_profile_enable(False)
    torch.cuda.synchronize()
    stages = {n: float(v) for n, v in zip(PREFILL_STAGES, np.array(stage_ms).mean(axis=0))}

    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    clk = ClockSampler(dev.index or 0) if with_clocks else None
    if clk:
        clk.__enter__()
    for i in range(steps):
        flush.zero_()
        ev0[i].record(stream)
        layer.prefill(x, out)
        ev1[i].record(stream)
    torch.cuda.synchronize()
    if clk:
        clk.__exit__()
    barrier(world)
    assert mka.mka_status() == 0
    step_ms = [a.elapsed_time(b) for a, b in zip(ev0, ev1)]
    value, ms = job_throughput(cfg.tokens, statistics.mean(step_ms), world)

    peaks = load_peaks()
    fl = prefill_flops(cfg)
    clocks = clk.summary() if clk else None
    res = {"value": round(value, 1), "unit": "tokens/s", "ms_per_step": round(ms, 4), "steps": steps,
           "roofline": attention_roofline(cfg, stages["attention"], peaks, sustained=power_capped(clocks)),
           "hbm": hbm_rooflines(cfg, stages, peaks),
           "layer_tflops": round((fl["projections"] + fl["attention"]) / (ms / 1e3) / 1e12, 1),
           "stage_ms": {n: round(v, 4) for n, v in stages.items()},
           "gpu_launches": prefill_kernels(cfg) * steps}
    if clk:
        res["clocks"] = clocks
    if with_e2e:
        res["e2e"] = measure_e2e(layer, inp, cfg, x, out, flush, world, max(4, steps))
    res["_recall_gpu"] = None
    if getattr(args, "recall_check", True) and cfg.tiers & 4 and cfg.attention_paths == 1:
        idx = torch.empty(cfg.batch, cfg.seq, cfg.recall_r, dtype=torch.int32, device=dev)
        layer.prefill(x, out, None, idx)
        torch.cuda.synchronize()
        assert mka.mka_status() == 0
        res["_recall_gpu"] = idx.cpu().numpy().astype(np.int64)
    del layer, x, out, flush, weights
    torch.cuda.empty_cache()
    return res, inp


def measure_e2e(layer, inp, cfg, x, out, flush, world, n_e2e):
    """End to end through host buffers (pinned): every step copies its X in (H2D), runs the layer and
    copies its O out (D2H), all inside the timed region.  Steps are pipelined the way a serving loop
    streams batches: three streams and double-buffered device X / O, so the copy-in of step i+1 and the
    copy-out of step i-1 (separate copy engines, full-duplex PCIe) overlap the layer of step i.  L2 is
    flushed before every layer call, as in the timed loop."""
    dev = x.device
    x_host = inp.x[:, :cfg.seq].contiguous().pin_memory()
    o_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    xb, ob = [x, torch.empty_like(x)], [out, torch.empty_like(out)]
    s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_cmp = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        t0.record(s_in)
        for i in range(n):
            k = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])   # layer i-2 has read xb[k]
                xb[k].copy_(x_host, non_blocking=True)
                ev_in[i].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[i])
                if i >= 2:
                    s_cmp.wait_event(ev_out[i - 2])  # ob[k] copied out
                flush.zero_()
                layer.prefill(xb[k], ob[k], stream=s_cmp)
                ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                o_host[k].copy_(ob[k], non_blocking=True)
                ev_out[i].record(s_out)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / n

    e2e_run(3)
    e2e_value, e2e_ms = job_throughput(cfg.tokens, e2e_run(n_e2e), world)
    return {"value": round(e2e_value, 1), "unit": "tokens/s",
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": o_host[0].numel() * o_host[0].element_size(), "ms_per_step": round(e2e_ms, 4),
            "steps": n_e2e,
            "how": "pinned host X -> device, layer, device O -> pinned host, every step; steps pipelined over "
                   "copy-in / compute / copy-out streams with double-buffered device X and O"}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = workload_cfg(args, args.workload)
    head, inp = measure_prefill(args, cfg, dev, world, args.steps, args.warmup, with_e2e=True, with_clocks=True)
    recall_gpu = head.pop("_recall_gpu")
    result = {
        "metric": "FastMKA layer prefill tokens/s (decode us/token and roofline fraction alongside)",
        "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic (seeded N(0,1) inputs, N(0,1/d_in) weights)",
        "config": workload_config(cfg, world),
        "roofline": head["roofline"],
        "hbm_roofline": head["hbm"],
        "layer_tflops": head["layer_tflops"],
        "stage_ms": head["stage_ms"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
    }
    others = [w for w in args.by_workload if w != cfg.name]
    if others:
        result["by_workload"] = {}
        for name in others:
            c = workload_cfg(args, name)
            r, _ = measure_prefill(args, c, dev, world, min(args.steps, 20), args.warmup)
            rec = r.pop("_recall_gpu")
            if rank == 0 and world == 1 and not args.no_cpu_baseline and rec is not None:
                r["recall"] = recall_check(c, make_inputs(c), rec)
            r["config"] = workload_config(c, world)["workload"]
            result["by_workload"][name] = r
    if world == 1 and not args.no_decode and args.paths == 1 and not args.block_sparse:  # prefill-only variants
        result["decode"] = run_decode(args, cfg, None, None, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(cfg, inp, prefix_tokens=args.cpu_prefix, attn_rows=args.cpu_rows)
        if recall_gpu is not None:
            result["recall"] = recall_check(cfg, inp, recall_gpu)
    return result


BACKWARD_STAGES = ["dsum", "attention_bwd", "router_preact_gemm", "router_bwd", "dq_gemm", "memory_adjoint", "dx_gemm",
                   "weight_grad_gemms"]


def train_flops(cfg) -> dict:
    """Algorithmic FLOPs of one training step (forward + backward).  Attention backward: the five
    products of the textbook backward over the causal pairs (S and dP recomputed once, dV, dK, dQ),
    10 dh Hq per pair; projections: dX and the weight gradients are two more GEMMs of the forward's
    size, plus the router's hidden layer recomputed and its two backward products."""
    fw = prefill_flops(cfg)
    pairs = cfg.batch * cfg.seq * (cfg.seq + 1) / 2
    T, d, dq, dkv, rh = cfg.tokens, cfg.d_model, cfg.dq, cfg.dkv, cfg.router_hidden
    return {"forward": fw["projections"] + fw["attention"],
            "attention_bwd": 10.0 * cfg.d_head * cfg.n_q_heads * pairs,
            "projections_bwd": 2.0 * T * d * (dq + 2 * dkv) * 2 + 2.0 * T * d * 2 * rh + 2.0 * T * dq * rh * 2}


def run_train(args, rank, world, local_rank):
    """Training step of the layer: mka_prefill_forward_train then mka_prefill_backward with a fixed
    synthetic output gradient; tokens/s of the whole step, roofline on the attention backward."""
    import route_kv_memory_b200 as mka
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    cfg = workload_cfg(args, args.workload)
    inp = make_inputs(cfg)
    weights = {k: v.to(dev) for k, v in inp.tensors().items() if k != "x"}
    layer = mka.FastMKALayer(cfg, weights, dev)
    x = inp.x[:, :cfg.seq].contiguous().to(dev)
    out = torch.empty(cfg.batch, cfg.seq, cfg.dq, dtype=x.dtype, device=dev)
    g = torch.Generator().manual_seed(cfg.seed + 1000)
    dout_host = torch.randn(cfg.batch, cfg.seq, cfg.dq, generator=g).to(torch.bfloat16)
    dout = dout_host.to(dev)
    f32 = dict(dtype=torch.float32, device=dev)
    grads = {"dx": torch.empty_like(x), "dw_q": torch.empty(cfg.d_model, cfg.dq, **f32),
             "dw_k": torch.empty(cfg.d_model, cfg.dkv, **f32), "dw_v": torch.empty(cfg.d_model, cfg.dkv, **f32),
             "dw_r1": torch.empty(cfg.dq, cfg.router_hidden, **f32), "dw_r2": torch.empty(cfg.router_hidden, 3, **f32)}
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step():
        layer.forward_train(x, out)
        layer.backward(x, out, dout, grads)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert mka.mka_status() == 0
    fw_ms, bw_ms = [], []
    mka.mka_profile_enable(True)
    for i in range(min(args.steps, 10)):
        flush.zero_()
        layer.forward_train(x, out)
        fw_ms.append(mka.mka_profile_read())
        layer.backward(x, out, dout, grads)
        bw_ms.append(mka.mka_profile_read(len(BACKWARD_STAGES)))
    mka.mka_profile_enable(False)
    torch.cuda.synchronize()
    fw_st, bw_st = np.array(fw_ms).mean(axis=0), np.array(bw_ms).mean(axis=0)

    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.zero_()
            ev0[i].record(stream)
            step()
            ev1[i].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    value, ms = job_throughput(cfg.tokens, statistics.mean(a.elapsed_time(b) for a, b in zip(ev0, ev1)), world)
    assert mka.mka_status() == 0

    # end to end: X and dO from pinned host memory, dX back, every step (sequential)
    x_host, dx_host = inp.x[:, :cfg.seq].contiguous().pin_memory(), torch.empty(x.shape, dtype=x.dtype).pin_memory()
    dout_pin = dout_host.pin_memory()
    n_e2e = max(4, args.steps // 4)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(n_e2e):
        x.copy_(x_host, non_blocking=True)
        dout.copy_(dout_pin, non_blocking=True)
        flush.zero_()
        step()
        dx_host.copy_(grads["dx"], non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    e2e_value, e2e_ms = job_throughput(cfg.tokens, t0.elapsed_time(t1) / n_e2e, world)

    peaks = load_peaks()
    fl = train_flops(cfg)
    ab_ms = float(bw_st[BACKWARD_STAGES.index("attention_bwd")])
    ab_tf = fl["attention_bwd"] / (ab_ms / 1e3) / 1e12
    return {
        "metric": "FastMKA layer training step (forward + backward) tokens/s",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) inputs and output gradient, N(0,1/d_in) weights)",
        "config": {"workload": f"{cfg.name}: {model_name(cfg)}-shaped FastMKA layer training step (forward keeping "
                               f"activations + backward to dX and dW_q, dW_k, dW_v, dW_r1, dW_r2), batch "
                               f"{cfg.batch} x seq {cfg.seq}; recall held fixed (straight-through)",
                   "global_batch": cfg.batch * world, "seq_len": cfg.seq,
                   "parallelism": f"replicas x{world} (independent sequences, no exchange)",
                   "l2": "flushed (512 MB write) before every timed step"},
        "roofline": {"kernel": "attention backward (dK/dV and dQ kernels)", "bound": "tensor",
                     "achieved": round(ab_tf, 1), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(ab_tf / peaks["bf16_tflops"], 4),
                     "peak_source": f"{peaks['source']} bf16 dense (burst, kernel timed per step)",
                     "traffic": traffic_from_profiles("attention_bwd", cfg.name),
                     "avg_ms": round(ab_ms, 4), "flops_per_launch": fl["attention_bwd"]},
        "layer_tflops": round(sum(fl.values()) / (ms / 1e3) / 1e12, 1),
        "forward_stage_ms": {n: round(float(v), 4) for n, v in zip(PREFILL_STAGES, fw_st)},
        "backward_stage_ms": {n: round(float(v), 4) for n, v in zip(BACKWARD_STAGES, bw_st)},
        "e2e": {"value": round(e2e_value, 1), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * x_host.numel() * x_host.element_size(),
                "d2h_bytes_per_step": dx_host.numel() * dx_host.element_size(), "ms_per_step": round(e2e_ms, 4),
                "how": "pinned host X and dO -> device, training step, device dX -> pinned host, sequential"},
        "gpu_launches": train_kernels() * args.steps,
        "clocks": clk.summary(),
    }


def train_kernels() -> int:
    """Kernel launches of one training step: the 10 of the prefill, then the backward's D, the two
    attention-backward kernels, the router pre-activation GEMM, the EMA and recalled-mean recomputes
    (2), the router backward, the dq GEMM (which adds the attention's dq in its epilogue), the recall
    lists (3), the memory adjoint (4), the dX GEMM and the two weight-gradient GEMMs (their operands
    read MN-major as stored, no transposes)."""
    return 10 + 1 + 2 + 1 + 2 + 1 + 1 + 3 + 4 + 1 + 2


def run_decode(args, cfg_prefill, inp_unused, weights_unused, dev, layer_pack=None):
    """Decode us/token over a fused cache of `ctx` positions: 256 steps captured in one CUDA graph."""
    import route_kv_memory_b200 as mka
    out = {}
    dcfg = workload_cfg(args, "qwen7b_decode")
    dinp = make_inputs(dcfg, seq_total=max(args.decode_ctx) + dcfg.decode_new)
    w = {k: v.to(dev) for k, v in dinp.tensors().items() if k != "x"}
    peaks = load_peaks()
    for ctx in args.decode_ctx:
        n_new = dcfg.decode_new
        lmax = ctx + n_new
        c = dcfg.replace(seq=ctx, decode_new=0)
        layer = mka.FastMKALayer(c, w, dev)
        x = dinp.x[:, :ctx + n_new].contiguous().to(dev)
        pre = torch.empty(1, ctx, dcfg.dq, dtype=x.dtype, device=dev)
        state = layer.new_state(lmax)
        layer.prefill(x[:, :ctx].contiguous(), pre, state=state, max_positions=lmax)
        snapshot = state.clone()
        xs = [x[:, t].contiguous() for t in range(ctx, ctx + n_new)]
        outs = [torch.empty(1, dcfg.dq, dtype=x.dtype, device=dev) for _ in range(n_new)]
        # per-stage times of one eager step (profiling off in the graph), after one warm-up step
        # (the first decode call of a process pays one-time launch set-up)
        layer.decode(state, lmax, xs[0], outs[0])
        state.copy_(snapshot)
        mka.mka_profile_enable(True)
        layer.decode(state, lmax, xs[0], outs[0])
        stages = mka.mka_profile_read()
        mka.mka_profile_enable(False)
        state.copy_(snapshot)
        torch.cuda.synchronize()
        s = torch.cuda.Stream(device=dev)
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(s):
            layer.decode(state, lmax, xs[0], outs[0], stream=s)  # creates the workspace outside capture
            state.copy_(snapshot)
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s):
                for t in range(n_new):
                    layer.decode(state, lmax, xs[t], outs[t], stream=s)
        torch.cuda.synchronize()
        times = []
        for rep in range(4):
            state.copy_(snapshot)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize()
            if rep > 0:
                times.append(e0.elapsed_time(e1))
        assert mka.mka_status() == 0
        us = statistics.mean(times) * 1e3 / n_new
        ntot = dcfg.dq + 2 * dcfg.dkv + 2 * dcfg.router_hidden + dcfg.hash_bits
        byt = decode_bytes_per_token(dcfg, ctx + n_new // 2, ntot)
        gbs = byt / (us * 1e-6) / 1e9
        out[str(ctx)] = {"us_per_token": round(us, 2), "tokens": n_new, "launches_per_token": 1,
                         "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                                      "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                                      "bytes_per_token": byt},
                         "fused_step_us_eager": round(stages[0] * 1e3, 2)}
        del g, layer, x, pre, state, snapshot, xs, outs
        torch.cuda.empty_cache()
    return {"workload": "qwen7b_decode: Qwen2.5-7B-shaped decode, batch 1, 256 new tokens after a prefilled "
                        "fused cache; block 256, R 8, nbits 32, alpha 0.99, seed 4",
            "kernel": "one cooperative launch per token: projection GEMV, token update + split-KV attention, merge",
            "timing": "256 steps in one CUDA graph, CUDA events around the replay, weights and cache resident",
            "by_context": out}


# ------------------------------------------------------------------ CPU oracle
def cpu_baseline(cfg, inp, prefix_tokens=8192, attn_rows=32):
    """The oracle as it stands on this host's cores, on a bounded sample of the workload: the whole
    layer over the first rows of every sequence (prefix_tokens in all; causality makes those rows
    exactly the full layer's first rows) with the attention on a strided sample of them, then
    extrapolated to the full workload: the linear parts (projections, router, EMA, L3, fuse, K/V)
    by token count, the attention by causal pair count."""
    import oracle
    P = max(cfg.block, min(cfg.seq, prefix_tokens // cfg.batch))
    c = cfg.replace(seq=P)
    X = inp.x[:, :P].float().numpy()
    w = oracle.weights_f64(*(to_f64(t) for t in (inp.w_q, inp.w_k, inp.w_v, inp.w_r1, inp.w_r2, inp.hash_proj)))
    rows = sample_rows(P, cfg.block, max_rows=attn_rows)
    t0 = time.perf_counter()
    out = oracle.fastmka_prefill(X, w, c, rows=rows)
    t_total = time.perf_counter() - t0
    t1 = time.perf_counter()
    for bi in range(cfg.batch):
        oracle.causal_gqa_attention(out["q"][bi], rows, out["K"][bi], out["V"][bi], cfg.n_kv_heads, cfg.scale)
    t_attn = time.perf_counter() - t1
    t_lin = max(t_total - t_attn, 0.0)
    pairs_all = cfg.seq * (cfg.seq + 1) / 2
    pairs_sample = float(np.sum(rows + 1))
    t_full = t_lin * cfg.seq / P + t_attn * pairs_all / pairs_sample
    cores = len(os.sched_getaffinity(0))
    return {"value": round(cfg.tokens / t_full, 3), "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "value_is": "extrapolated from the measured sample to the whole workload",
            "sample": f"float64 NumPy oracle, {cfg.name}: the layer over the first {P} rows of each of {cfg.batch} "
                      f"sequence(s) ({t_lin:.2f} s for projections/router/EMA/L3/fuse/K,V) with the attention on "
                      f"{len(rows)} strided rows per sequence ({t_attn:.2f} s); extrapolated by token count "
                      f"(x{cfg.seq / P:.0f}) and causal pair count (x{pairs_all / pairs_sample:.0f}) to "
                      f"{t_full:.0f} s per layer",
            "measured_s": round(t_total, 2)}


def recall_check(cfg, inp, idx_gpu, max_rows=16384):
    """The GPU's recalled block indices against the oracle's L3 recall on the same inputs: every
    row for workloads up to max_rows tokens per sequence, else a strided row sample.  A mismatch is
    excused only where the GPU's list is the recall under a flip of hash bits within 1e-4 of zero."""
    import oracle
    P = to_f64(inp.hash_proj)
    S, b = cfg.seq, cfg.block
    stride = max(1, -(-S // max_rows))
    rows = np.arange(0, S, stride)
    nblk = S // b
    t0 = time.perf_counter()
    ref = {"idx": np.full((cfg.batch, len(rows), cfg.recall_r), -1, np.int64), "block": b,
           "x_proj": np.zeros((cfg.batch, S, P.shape[1])), "summary_proj": np.zeros((cfg.batch, nblk, P.shape[1]))}
    for bi in range(cfg.batch):
        summ = np.zeros((nblk, cfg.d_model))
        for j0 in range(0, nblk, 64):  # block means, 64 blocks of rows widened at a time
            j1 = min(nblk, j0 + 64)
            summ[j0:j1] = oracle.block_summaries(to_f64(inp.x[bi:bi + 1, j0 * b:j1 * b]), b)[0]
        xr = to_f64(inp.x[bi, :S][torch.from_numpy(rows)])
        idx, _, _, _, xproj = oracle.longterm_recall(xr, rows, summ, P, b, cfg.recall_r)
        ref["idx"][bi] = idx
        ref["x_proj"][bi, rows] = xproj
        ref["summary_proj"][bi] = oracle.hash_codes(summ, P)[1]
    full_ref = dict(ref, idx=np.full((cfg.batch, S, cfg.recall_r), -1, np.int64))
    full_ref["idx"][:, rows] = ref["idx"]
    unexcused, excused, _ = oracle.recall_mismatches(idx_gpu[:, rows], full_ref, rows)
    return {"rows_checked": int(cfg.batch * len(rows)), "rows_total": int(cfg.tokens),
            "rows": "all" if stride == 1 else f"every {stride}th row of each sequence",
            "mismatches_unexcused": unexcused, "mismatches_excused": excused,
            "rule": "bit-exact; excused only where a flip of hash bits with |p| < 1e-4 gives the GPU's list",
            "oracle_s": round(time.perf_counter() - t0, 1)}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle, timed per step on a bounded sample of the same workload."""
    if rank != 0:
        return None
    cfg = workload_cfg(args, args.workload)
    inp = make_inputs(cfg)
    vals = []
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(cfg, inp, prefix_tokens=args.ref_prefix, attn_rows=max(4, args.cpu_rows // 4))
        if i >= args.warmup:
            vals.append(r)
    v = statistics.mean(r["value"] for r in vals)
    ms = statistics.mean(r["measured_s"] for r in vals) * 1e3
    return {"impl": "reference", "metric": "FastMKA layer prefill tokens/s (decode us/token and roofline fraction "
                                           "alongside)", "value": round(v, 3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(cfg, world),
            "value_is": "tokens/s of the whole workload, extrapolated from each step's measured sample; "
                        "ms_per_step is the measured time of one sampled step",
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": vals[-1]["cores"], "kind": "oracle",
                             "sample": vals[-1]["sample"]},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def traffic_from_profiles(kernel: str, workload: str = None):
    """DRAM bytes (read + write) per launch of `kernel` at `workload` from the committed ncu summary
    profiles/traffic.txt; None when there is no capture of that workload or the kernel's source
    changed after the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel)
    if not d:
        return None
    with open(os.path.join(ROOT, d["source"]), "rb") as f:
        if hashlib.sha1(f.read()).hexdigest() != d["source_sha1"]:
            return None
    per = d["dram_bytes_per_launch"]
    return per.get(workload) if isinstance(per, dict) else per


# ------------------------------------------------------------------ distributed plumbing
def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int) -> float:
    """The largest of the ranks' values, returned on every rank.  The collective's tensor lives where
    the process group's backend wants it: on the GPU for NCCL, in host memory for gloo."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms: float, world: int):
    """Whole-job units per second and the job's time per step: every rank processes units_per_rank
    in its own `ms`, and the job takes as long as its slowest rank.  Returns (units/s, max ms)."""
    ms_max = max_over_ranks(ms, world)
    return world * units_per_rank / (ms_max / 1e3), ms_max


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=None,
                    help="the headline workload (default: llama8b_128k, the largest single-GPU prefill; "
                         "qwen7b_4k with --train)")
    ap.add_argument("--by-workload", nargs="*", default=["tiny_f32", "qwen7b_4k", "qwen7b_32k"],
                    help="further prefill workloads reported under by_workload (none: pass the flag alone)")
    ap.add_argument("--route", default="soft", choices=["soft", "fixed", "top1", "top2"],
                    help="routing gate variant (the published layer is soft)")
    ap.add_argument("--tiers", type=int, default=7, help="memory tier mask: 1 L1, 2 L2, 4 L3 (7 = all)")
    ap.add_argument("--paths", type=int, default=1, choices=[1, 3],
                    help="1: FastMKA (the layer measured); 3: full MKA, three attention paths (prefill only)")
    ap.add_argument("--block-sparse", action="store_true",
                    help="Block-MKA block-sparse attention: own block + recalled blocks (prefill only)")
    ap.add_argument("--train", action="store_true",
                    help="time the layer training step (forward keeping activations + backward) instead of prefill")
    ap.add_argument("--decode-ctx", type=int, nargs="*", default=[4096, 32768, 131072, 262144])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-only", action="store_true", help="run only the decode measurement (no prefill line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-rows", type=int, default=32, help="oracle attention rows per sequence in its sample")
    ap.add_argument("--cpu-prefix", type=int, default=8192, help="tokens of the oracle's prefix sample (main arm)")
    ap.add_argument("--ref-prefix", type=int, default=2048, help="tokens of each reference-arm step's prefix sample")
    ap.add_argument("--no-recall-check", dest="recall_check", action="store_false")
    ap.add_argument("--seq", type=int, default=None,
                    help="profiling: run the headline workload's shape at this sequence length instead")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.workload is None:
        args.workload = "qwen7b_4k" if args.train else "llama8b_128k"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.decode_only:
            torch.cuda.set_device(local_rank)
            dev = torch.device("cuda", local_rank)
            res = {"decode": run_decode(args, None, None, None, dev)}
            if rank == 0:
                print(json.dumps(res), flush=True)
            return
        res = run_train(args, rank, world, local_rank) if args.train else run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
