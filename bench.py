"""Benchmark: attention forward/backward TFLOP/s on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over the long-sequence head-dim-128
workload (B=2, Hq=Hkv=16, N=8192, d=128, causal, bf16 inputs drawn i.i.d.
N(0,1)): the forward (O and LSE) and, once built, the recompute backward.
FLOPs follow the workload statement: 4*B*Hq*N^2*d for the forward, halved for
the causal mask, and 2.5x that for the backward. Inputs (3 x 64 MiB) are
larger than the 126 MB L2, so no flush runs between steps.

Multi-GPU: every (batch, head) is an independent problem, so ranks run the
same per-GPU workload with no collective on the data path (weak scaling); the
value is all ranks' FLOPs over the slowest rank's device time.

``--impl reference`` times the fp64 CPU oracle (the only other
implementation: the pages ship no code) on a bounded sample of the same
workload, on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from synthetic import WORKLOADS, attention_inputs, bf16_bits_to_f32  # noqa: E402

WORKLOAD = "long128"
CAUSAL = True
PASSES = ("fwd",)
METRIC = "attention fwd/bwd TFLOP/s and % of B200 dense BF16/FP8 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def step_flops(w, passes=PASSES):
    f = 0.0
    if "fwd" in passes:
        f += w.fwd_flops(CAUSAL)
    if "bwd" in passes:
        f += w.bwd_flops(CAUSAL)
    return f


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = f"/tmp/.fa_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        self.f.close()

    def summary(self):
        try:
            rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
            os.remove(self.path)
        except Exception:
            return None
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if len(r) > 5 + i and "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def cpu_oracle_sample(w, seconds_budget=15.0):
    """Time the fp64 oracle on whole heads of the workload (head 0 of batch 0
    first, then further heads) until the budget is spent; returns
    (TFLOP/s, flops done, seconds, heads)."""
    import oracle
    try:
        import threadpoolctl
        threads = max(v["num_threads"] for v in threadpoolctl.threadpool_info()) if threadpoolctl.threadpool_info() else os.cpu_count()
    except Exception:
        threads = os.cpu_count()
    bits = attention_inputs(1, 1, 1, w.N, w.d, w.seed, with_dout=True)
    x = {n: bf16_bits_to_f32(a).astype(np.float64) for n, a in bits.items()}
    per_head = step_flops(w) / (w.B * w.Hq)
    done, heads, t0 = 0.0, 0, time.perf_counter()
    while True:
        oracle.attention_forward(x["q"], x["k"], x["v"], CAUSAL, w.scale)
        if "bwd" in PASSES:
            oracle.attention_backward(x["q"], x["k"], x["v"], x["do"], CAUSAL, w.scale)
        heads += 1
        done += per_head
        el = time.perf_counter() - t0
        if el > seconds_budget or heads >= 64:
            break
    return done / el / 1e12, done, el, heads, threads


def run_reference(args, rank, world):
    if rank != 0:
        return
    w = WORKLOADS[WORKLOAD]
    for _ in range(args.warmup):
        pass  # the oracle has no warm-up state; steps below are all timed
    vals = []
    t_all = 0.0
    heads_all = 0
    threads = os.cpu_count()
    budget = max(2.0, 60.0 / max(1, args.steps))
    for _ in range(args.steps):
        v, _, el, heads, threads = cpu_oracle_sample(w, seconds_budget=budget)
        vals.append(v)
        t_all += el
        heads_all += heads
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_all / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={CAUSAL}",
                   "passes": list(PASSES), "l2": "inputs larger than L2"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{heads_all} whole (batch, head) problems of the workload over {args.steps} steps"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import exact_tiled_attention_42_b200 as fa
    from exact_tiled_attention_42_b200 import _lib

    torch.cuda.set_device(local_rank)
    _lib.load()
    w = WORKLOADS[WORKLOAD]
    bits = attention_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, with_dout=("bwd" in PASSES))
    host = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for n, a in bits.items()}
    dev = {n: t.cuda() for n, t in host.items()}
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=CAUSAL, out=o, lse=lse)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0

    # --- device-timed region: K steps, per-launch events for the forward kernel
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t_start.elapsed_time(t_end)
    fwd_ms = [a.elapsed_time(b) for a, b in ev]
    clocks = clk.summary()
    if world > 1:
        t = torch.tensor([ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    flops = step_flops(w)
    value = world * flops * args.steps / (ms * 1e-3) / 1e12

    # --- end to end through the public API with pinned host buffers
    o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    lse_host = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(host[n].numel() * 2 for n in ("q", "k", "v"))
    d2h = o_host.numel() * 2 + lse_host.numel() * 4
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        for n in ("q", "k", "v"):
            dev[n].copy_(host[n], non_blocking=True)
        step()
        o_host.copy_(o, non_blocking=True)
        lse_host.copy_(lse, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device="cuda")
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = world * flops * args.steps / (e2e_ms * 1e-3) / 1e12

    if rank != 0:
        return
    pk, pk_kind = peaks()
    peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
    avg_fwd_ms = statistics.mean(fwd_ms)
    achieved = w.fwd_flops(CAUSAL) / (avg_fwd_ms * 1e-3) / 1e12
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, done, el, heads, threads = cpu_oracle_sample(w, seconds_budget=args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{heads} whole (batch, head) problem(s) of the workload, fp64 numpy, {el:.1f} s"}
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={CAUSAL}",
                   "passes": list(PASSES), "l2": "inputs larger than L2 (192 MiB of Q/K/V), no flush",
                   "parallelism": f"replica x{world} (independent problems per GPU)"},
        "fwd_tflops": achieved, "fwd_frac_of_peak": achieved / peak,
        "roofline": {"bound": "tensor", "kernel": "fwd_bf16_kernel", "achieved": achieved, "peak": peak,
                     "peak_kind": f"{pk_kind} bf16 dense, sustained", "unit": "TFLOP/s", "frac": achieved / peak,
                     "traffic": None},
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": args.steps * len(PASSES),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
