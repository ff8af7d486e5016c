"""Benchmark: attention forward/backward TFLOP/s on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over the long-sequence head-dim-128
workload (B=2, Hq=Hkv=16, N=8192, d=128, causal, bf16 inputs drawn i.i.d.
N(0,1)): the forward (O and LSE) and the recompute backward (dQ, dK, dV).
FLOPs follow the workload statement: 4*B*Hq*N^2*d for the forward, halved for
the causal mask, and 2.5x that for the backward. Inputs (3 x 64 MiB) are
larger than the 126 MB L2, so no flush runs between steps.

The JSON line also carries: `e2e`, the same step through the public API with
every step's inputs copied from pinned host memory and all results read back
(three streams, two buffer sets: neighbouring steps' copies overlap the
kernels); `fp8`, the FP8 workload's pre-pass + forward in TFLOP/s (and the
MXFP8 forward on the same inputs); `decode`,
one decode step (a query row per head against a 16K-key cache) in GB/s against
the measured HBM copy bandwidth; `workloads`, the other bf16 workloads (GQA
32/8 heads at N = 8192, d = 64 at N = 2048 causal and not, and the tiny
N = 128 case in GB/s); `roofline`, the dominant kernel against its peak.

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
PASSES = ("fwd", "bwd")
METRIC = "attention fwd/bwd TFLOP/s and % of B200 dense BF16/FP8 tensor peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


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


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic.json")


def sources_sha256(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(key: str):
    """DRAM bytes per launch that ncu measured for `key` (an entry of
    profiles/dram_traffic.json), or None when there is no entry or the kernel
    sources have changed since the counters were taken (each entry keeps the
    sha256 of the sources it was measured on)."""
    try:
        entries = json.load(open(TRAFFIC_FILE))["entries"]
    except (OSError, ValueError, KeyError):
        return None
    for e in entries:
        if e.get("key") != key:
            continue
        try:
            if sources_sha256(e["sources"]) == e["sha256"]:
                return float(e["bytes_per_launch"])
        except (OSError, KeyError, TypeError, ValueError):
            return None
    return None


BURST_REGION_MS = 1000.0


def choose_peak(pk: dict, region_ms: float, clocks) -> tuple:
    """The tensor peak a kernel is held to: the burst GEMM figure when the
    timed region is short (under a second) or the SM clock stayed at its
    maximum, the sustained (power-capped) figure otherwise. Returns (peak,
    which) with which = "burst" or "sustained"."""
    burst = pk["bf16_tflops"]
    sustained = pk.get("bf16_tflops_sustained", burst)
    at_max = False
    if clocks and clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        at_max = clocks["sm_mhz"] >= 0.97 * clocks["sm_max_mhz"]
    if region_ms < BURST_REGION_MS or at_max:
        return burst, "burst"
    return sustained, "sustained"


def max_over_ranks(x: float, world: int, device="cuda") -> float:
    """The largest of every rank's x (device time is reported as the slowest
    rank's). A no-op on one rank."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs the same per-GPU work, so the job did
    world x steps x flops in the slowest rank's time."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def _oracle_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(v["num_threads"] for v in info) if info else os.cpu_count()
    except Exception:
        return os.cpu_count()


def _host_info(threads) -> dict:
    """The host the oracle ran on: CPU model, logical CPUs, BLAS threads."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "logical_cpus": os.cpu_count(), "blas_threads": threads}


def _oracle_inputs(w):
    bits = attention_inputs(1, 1, 1, w.N, w.d, w.seed, with_dout=True)
    return {n: bf16_bits_to_f32(a).astype(np.float64) for n, a in bits.items()}


def _oracle_rows(x, w, causal, passes, rows):
    """One oracle sample: query rows ``rows`` of one (batch, head) problem."""
    import oracle
    oracle.attention_forward(x["q"], x["k"], x["v"], causal, w.scale, rows=rows)
    if "bwd" in passes:
        oracle.attention_backward(x["q"], x["k"], x["v"], x["do"], causal, w.scale, rows=rows)


def _sample_flops(w, causal, passes, nrows):
    """The workload's FLOP formula, per (batch, head), scaled to nrows rows."""
    per_head = sum((w.fwd_flops(causal) if p_ == "fwd" else w.bwd_flops(causal)) for p_ in passes) / (w.B * w.Hq)
    return per_head * nrows / w.N


def cpu_oracle_sample(w, causal, passes, seconds_budget=15.0):
    """Time the fp64 oracle on whole (batch, head) problems of the workload
    until the budget is spent; returns (TFLOP/s, seconds, problems, threads)."""
    x = _oracle_inputs(w)
    done, heads, t0 = 0.0, 0, time.perf_counter()
    while True:
        _oracle_rows(x, w, causal, passes, None)
        heads += 1
        done += _sample_flops(w, causal, passes, w.N)
        el = time.perf_counter() - t0
        if el > seconds_budget or heads >= 64:
            break
    return done / el / 1e12, el, heads, _oracle_threads()


def run_reference(args, rank, world):
    """The oracle as it stands, on the host cores: each step is a block of
    query rows around the middle of one (batch, head) problem (under a causal
    mask their cost is the average row's), sized so that the K steps take
    about a minute in total."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    causal = w.causal[0]
    passes = PASSES
    x = _oracle_inputs(w)
    # warm-up samples also calibrate the seconds per row
    r_cal = min(64, w.N)
    mid = w.N // 2
    t_row = None
    for _ in range(args.warmup):
        t0 = time.perf_counter()
        _oracle_rows(x, w, causal, passes, (mid - r_cal // 2, mid - r_cal // 2 + r_cal))
        t_row = (time.perf_counter() - t0) / r_cal
    per_step = max(0.05, 60.0 / max(1, args.steps))
    nrows = int(max(1, min(w.N, per_step / max(t_row, 1e-9))))
    r0 = max(0, mid - nrows // 2)
    rows = (r0, r0 + nrows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_rows(x, w, causal, passes, rows)
        times.append(time.perf_counter() - t0)
    t_step = statistics.mean(times)
    value = _sample_flops(w, causal, passes, nrows) / t_step / 1e12
    threads = _oracle_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={causal}",
                   "passes": list(passes), "l2": "inputs larger than L2 (no flush between steps)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: query rows {rows[0]}..{rows[1] - 1} of one (batch, head) problem, "
                                   f"fp64 numpy oracle, {len(passes)} pass(es)",
                         "host": _host_info(threads)},
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
    w = WORKLOADS[args.workload]
    causal = w.causal[0]
    passes = PASSES
    bits = attention_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, with_dout=("bwd" in passes))
    host = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).pin_memory() for n, a in bits.items()}
    dev = {n: t.cuda() for n, t in host.items()}
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    o = torch.empty_like(dev["q"])
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()

    dq = torch.empty_like(dev["q"])
    dk = torch.empty_like(dev["k"])
    dv = torch.empty_like(dev["v"])
    ws = torch.empty(fa.fa_bwd_workspace_size(B, Hq, Hkv, N, d), dtype=torch.uint8, device="cuda")

    def fwd():
        fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal, out=o, lse=lse)

    def bwd():
        fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal, dq=dq, dk=dk, dv=dv,
                  workspace=ws)

    def step():
        fwd()
        if "bwd" in passes:
            bwd()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert fa.fa_last_device_status() == 0

    # --- device-timed region: K steps; events around each pass on the
    # launching stream give the per-launch duration of each kernel
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        time.sleep(0.5)  # let nvidia-smi start sampling before the timed region
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            fwd()
            ev[i][1].record(stream)
            if "bwd" in passes:
                bwd()
            ev[i][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = t_start.elapsed_time(t_end)
    fwd_ms = [a.elapsed_time(b_) for a, b_, _ in ev]
    bwd_ms = [b_.elapsed_time(c) for _, b_, c in ev]
    clocks = clk.summary()
    ms = max_over_ranks(ms, world)
    flops = sum((w.fwd_flops(causal) if p_ == "fwd" else w.bwd_flops(causal)) for p_ in passes)
    value = weak_scaling_value(flops, args.steps, world, ms)

    # --- end to end through the public API with pinned host buffers: every
    # step copies its inputs host->device and reads O, LSE (and dQ, dK, dV)
    # back. Three streams and two device buffer sets: step i's kernels run
    # while step i+1's inputs arrive and step i-1's results leave (the host
    # link is full duplex), the way a pipeline of independent problems runs.
    e2e = None
    if not args.no_e2e:
        e2e_steps = min(args.steps, 50)
        ins = [n for n in ("q", "k", "v", "do") if n in host]
        bufs = []
        for _ in range(2):
            bi = {n: torch.empty_like(dev[n]) for n in ins}
            bo = {"o": torch.empty_like(o), "lse": torch.empty_like(lse)}
            if "bwd" in passes:
                bo.update(dq=torch.empty_like(dq), dk=torch.empty_like(dk), dv=torch.empty_like(dv))
            bufs.append((bi, bo))
        out_host = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in bufs[0][1].items()}
        h2d = sum(host[n].numel() * 2 for n in ins)
        d2h = sum(h.numel() * h.element_size() for h in out_host.values())
        s_in, s_run, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_ready, run_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]

        def e2e_step(i):
            bi, bo = bufs[i & 1]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(run_done[i & 1])  # step i-2 has finished reading these inputs
                for n in ins:
                    bi[n].copy_(host[n], non_blocking=True)
                in_ready[i & 1].record(s_in)
            s_run.wait_event(in_ready[i & 1])
            if i >= 2:
                s_run.wait_event(out_done[i & 1])  # step i-2's results have left these buffers
            fa.fa_fwd(bi["q"], bi["k"], bi["v"], causal=causal, out=bo["o"], lse=bo["lse"], stream=s_run)
            if "bwd" in passes:
                fa.fa_bwd(bi["q"], bi["k"], bi["v"], bo["o"], bo["lse"], bi["do"], causal=causal, dq=bo["dq"],
                          dk=bo["dk"], dv=bo["dv"], workspace=ws, stream=s_run)
            run_done[i & 1].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(run_done[i & 1])
                for n, h in out_host.items():
                    h.copy_(bo[n], non_blocking=True)
                out_done[i & 1].record(s_out)

        for i in range(2):  # warm the streams and buffers
            e2e_step(i)
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_run.wait_event(e0)
        s_out.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        s_in.wait_event(out_done[(e2e_steps - 1) & 1])
        e1.record(s_in)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": weak_scaling_value(flops, e2e_steps, world, e2e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
               "overlap": "3 streams, 2 buffer sets: copies of neighbouring steps overlap the kernels"}
    assert fa.fa_last_device_status() == 0

    fp8 = None if args.no_fp8 else run_fp8_leg(args, fa, stream)
    decode = None if args.no_decode else run_decode_leg(args, fa, stream)
    assert fa.fa_last_device_status() == 0

    workloads = None if args.no_workloads else run_workloads_leg(args, fa, stream)
    assert fa.fa_last_device_status() == 0

    if rank != 0:
        return
    pk, pk_kind = peaks()
    peak, which = choose_peak(pk, ms, clocks)
    fwd_tf = w.fwd_flops(causal) / (statistics.mean(fwd_ms) * 1e-3) / 1e12
    bwd_tf = w.bwd_flops(causal) / (statistics.mean(bwd_ms) * 1e-3) / 1e12 if "bwd" in passes else None
    # dominant kernel: the backward (2.5x the forward's FLOPs); its events
    # bracket the whole fa_bwd call (preprocess + main + postprocess), so the
    # figure is a lower bound for the main kernel alone
    if "bwd" in passes:
        dom, achieved = "fa_bwd: bwd_pre_kernel + bwd_bf16_kernel + bwd_post_kernel", bwd_tf
        traffic = recorded_traffic(f"fa_bwd {args.workload}")
    else:
        dom, achieved = "fwd_bf16_kernel", fwd_tf
        traffic = recorded_traffic(f"fwd_bf16_kernel {args.workload}")
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v, el, heads, threads = cpu_oracle_sample(w, causal, passes, seconds_budget=args.cpu_seconds)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": f"{heads} whole (batch, head) problem(s) of the workload, fp64 numpy, {el:.1f} s",
               "host": _host_info(threads)}
    peak_note = (f"{pk_kind} bf16 dense, {which} (timed region {ms:.0f} ms, median SM clock "
                 f"{clocks.get('sm_mhz') if clocks else None} of {clocks.get('sm_max_mhz') if clocks else None} MHz; "
                 f"burst below {BURST_REGION_MS:.0f} ms or at the maximum clock, sustained otherwise)")
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"{args.workload}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={causal}",
                   "passes": list(passes), "l2": "inputs larger than L2 (no flush between steps)",
                   "parallelism": f"replica x{world} (independent problems per GPU)"},
        "fwd_tflops": fwd_tf, "fwd_frac_of_peak": fwd_tf / peak,
        "bwd_tflops": bwd_tf, "bwd_frac_of_peak": (bwd_tf / peak) if bwd_tf else None,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "peak_kind": peak_note, "peak_burst": pk["bf16_tflops"],
                     "peak_sustained": pk.get("bf16_tflops_sustained"),
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "workloads": workloads,
        "fp8": fp8,
        "decode": decode,
        "gpu_launches": args.steps * (1 + (3 if "bwd" in passes else 0)),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def _time_calls(fn, calls, warmup, stream):
    """Mean device milliseconds per call: CUDA events around each call on the
    launching stream, after `warmup` untimed calls."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(calls)]
    for a, b_ in ev:
        a.record(stream)
        fn()
        b_.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b_) for a, b_ in ev)


def run_workloads_leg(args, fa, stream):
    """The other bf16 workloads, forward and backward timed apart: gqa
    (B=2, Hq=32, Hkv=8, N=8192, d=128, causal) and gpt2 (B=8, H=16, N=2048,
    d=64, causal and not) in TFLOP/s against the tensor peak; tiny (B=1, H=2,
    N=128, d=64) in GB/s of algorithmic bytes against the HBM copy bandwidth
    (at N = 128 nothing keeps the tensor cores busy: the call is bound by
    launch latency and memory)."""
    import torch
    pk, pk_kind = peaks()
    out = {}
    for name, causal, calls in (("gqa", True, 20), ("gpt2", True, 50), ("gpt2", False, 50),
                                ("tiny", False, 200), ("tiny", True, 200)):
        w = WORKLOADS[name]
        bits = attention_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, with_dout=True)
        dev = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for n, a in bits.items()}
        o = torch.empty_like(dev["q"])
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
        dq, dk, dv = torch.empty_like(dev["q"]), torch.empty_like(dev["k"]), torch.empty_like(dev["v"])
        ws = torch.empty(fa.fa_bwd_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8, device="cuda")
        fwd = lambda: fa.fa_fwd(dev["q"], dev["k"], dev["v"], causal=causal, out=o, lse=lse)
        bwd = lambda: fa.fa_bwd(dev["q"], dev["k"], dev["v"], o, lse, dev["do"], causal=causal, dq=dq, dk=dk,
                                dv=dv, workspace=ws)
        f_ms = _time_calls(fwd, calls, args.warmup, stream)
        b_ms = _time_calls(bwd, calls, args.warmup, stream)
        key = f"{name}_{'causal' if causal else 'noncausal'}"
        desc = f"{name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={causal}"
        if name == "tiny":
            q_el, kv_el = dev["q"].numel(), dev["k"].numel()
            fwd_bytes = 2 * (2 * q_el + 2 * kv_el) + 4 * lse.numel()          # Q, K, V read; O written; LSE
            bwd_bytes = 2 * (4 * q_el + 4 * kv_el) + 4 * lse.numel()          # Q, K, V, O, dO; dQ, dK, dV; LSE
            gf, gb = fwd_bytes / (f_ms * 1e-3) / 1e9, bwd_bytes / (b_ms * 1e-3) / 1e9
            out[key] = {"workload": desc, "bound": "hbm / launch latency", "fwd_us": f_ms * 1e3, "bwd_us": b_ms * 1e3,
                        "fwd_gbs": gf, "bwd_gbs": gb, "fwd_bytes": fwd_bytes, "bwd_bytes": bwd_bytes,
                        "peak_gbs": pk["hbm_gbs"], "fwd_frac_of_peak": gf / pk["hbm_gbs"],
                        "bwd_frac_of_peak": gb / pk["hbm_gbs"], "calls": calls}
        else:
            peak, which = choose_peak(pk, calls * (f_ms + b_ms), None)
            ft = w.fwd_flops(causal) / (f_ms * 1e-3) / 1e12
            bt = w.bwd_flops(causal) / (b_ms * 1e-3) / 1e12
            out[key] = {"workload": desc, "bound": "tensor", "fwd_tflops": ft, "bwd_tflops": bt,
                        "fwd_frac_of_peak": ft / peak, "bwd_frac_of_peak": bt / peak, "peak": peak,
                        "peak_kind": f"{pk_kind} bf16 dense, {which}", "calls": calls,
                        "fwd_ms": f_ms, "bwd_ms": b_ms}
        del dev, o, lse, dq, dk, dv, ws
    torch.cuda.empty_cache()
    return out


def run_fp8_leg(args, fa, stream):
    """The FP8 forward on its own workload (B=1, H=16, N=16384, d=128,
    non-causal, 0.1% entry outliers), timed with events around each
    fa_fwd_fp8 call (quantisation pre-pass + FP8 forward)."""
    import torch
    w = WORKLOADS["fp8"]
    causal = w.causal[0]
    bits = attention_inputs(w.B, w.Hq, w.Hkv, w.N, w.d, w.seed, outlier_rate=w.outlier_rate, with_dout=False)
    dev = {n: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for n, a in bits.items()}
    o = torch.empty_like(dev["q"])
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_fp8_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8, device="cuda")

    def call():
        fa.fa_fwd_fp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=w.seed, use_rotation=True,
                      out=o, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 300))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b_ in ev:
        a.record(stream)
        call()
        b_.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b_) for a, b_ in ev)
    # the FP8 forward alone, from a workspace quantised once
    fa.fa_fp8_quantize(dev["q"], dev["k"], dev["v"], rotation_seed=w.seed, use_rotation=True, workspace=ws)
    shape = (w.B, w.Hq, w.Hkv, w.N, w.d)

    def call_fwd_only():
        fa.fa_fwd_fp8_quantized(ws, shape, causal=causal, use_rotation=True, out=o, lse=lse)

    for _ in range(args.warmup):
        call_fwd_only()
    torch.cuda.synchronize()
    for a, b_ in ev:
        a.record(stream)
        call_fwd_only()
        b_.record(stream)
    torch.cuda.synchronize()
    ms_k = statistics.mean(a.elapsed_time(b_) for a, b_ in ev)
    # the MXFP8 forward (32-element E8M0 block scales applied by the tensor
    # cores; pre-pass + forward in one call), same inputs
    ws_mx = torch.empty(fa.fa_mxfp8_workspace_size(w.B, w.Hq, w.Hkv, w.N, w.d), dtype=torch.uint8, device="cuda")

    def call_mx():
        fa.fa_fwd_mxfp8(dev["q"], dev["k"], dev["v"], causal=causal, rotation_seed=w.seed, use_rotation=True,
                        scale_rule="fit", out=o, lse=lse, workspace=ws_mx)

    for _ in range(args.warmup):
        call_mx()
    torch.cuda.synchronize()
    for a, b_ in ev:
        a.record(stream)
        call_mx()
        b_.record(stream)
    torch.cuda.synchronize()
    ms_mx = statistics.mean(a.elapsed_time(b_) for a, b_ in ev)
    pk, pk_kind = peaks()
    bf16_peak, which = choose_peak(pk, steps * (ms + ms_k + ms_mx), None)
    fp8_peak = 2.0 * bf16_peak
    tf = w.fwd_flops(causal) / (ms * 1e-3) / 1e12
    tf_k = w.fwd_flops(causal) / (ms_k * 1e-3) / 1e12
    tf_mx = w.fwd_flops(causal) / (ms_mx * 1e-3) / 1e12
    return {"workload": f"fp8: B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} causal={causal} e4m3",
            "tflops": tf, "ms_per_call": ms, "calls": steps,
            "kernel_only_tflops": tf_k, "kernel_only_ms": ms_k,
            "peak": fp8_peak, "peak_kind": f"nominal: {pk_kind} bf16 dense {which} x 2 (the datasheet's fp8:bf16 "
                                              "ratio; no fp8 peak is measured)",
            "frac_of_peak": tf / fp8_peak, "kernel_only_frac_of_peak": tf_k / fp8_peak,
            "mxfp8_tflops": tf_mx, "mxfp8_ms_per_call": ms_mx, "mxfp8_frac_of_peak": tf_mx / fp8_peak,
            "includes": "tflops: quantisation pre-pass (Hadamard rotation, 64-row block scales) + FP8 forward; "
                        "kernel_only: the FP8 forward from an already quantised workspace; "
                        "mxfp8: fa_fwd_mxfp8 (rule fit: MX pre-pass + MXFP8 forward)"}


def run_decode_leg(args, fa, stream):
    """Decode step (one query row per head against a 16K-key cache, GQA 32/8),
    timed with events around each fa_fwd_decode call (split pass + combine).
    HBM-bound: reported in GB/s of algorithmic bytes (K, V, Q read; O, LSE
    written) against the measured copy bandwidth. K and V (1.07 GB) exceed L2."""
    import torch
    w = WORKLOADS["decode"]
    causal = w.causal[0]
    kv = attention_inputs(w.B, w.Hkv, w.Hkv, w.N, w.d, w.seed, with_dout=False)
    qq = attention_inputs(w.B, w.Hq, w.Hq, w.nq, w.d, w.seed + 1000, with_dout=False)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = to_dev(qq["q"]), to_dev(kv["k"]), to_dev(kv["v"])
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.nq), dtype=torch.float32, device="cuda")
    ws = torch.empty(fa.fa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.nq, w.N, w.d, 0), dtype=torch.uint8,
                     device="cuda")

    def call():
        fa.fa_fwd_decode(q, k, v, causal=causal, out=o, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 500))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b_ in ev:
        a.record(stream)
        call()
        b_.record(stream)
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b_) for a, b_ in ev)
    nbytes = (k.numel() + v.numel() + q.numel() + o.numel()) * 2 + lse.numel() * 4
    gbs = nbytes / (ms * 1e-3) / 1e9
    pk, pk_kind = peaks()
    return {"workload": f"decode: B={w.B} Hq={w.Hq} Hkv={w.Hkv} Nq={w.nq} Nk={w.N} d={w.d} causal={causal}",
            "gbs": gbs, "us_per_call": ms * 1e3, "calls": steps, "bytes_per_call": nbytes,
            "peak_gbs": pk["hbm_gbs"], "peak_kind": f"{pk_kind} HBM copy bandwidth", "frac_of_peak": gbs / pk["hbm_gbs"],
            "includes": "split pass over the keys + log-sum-exp combine"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg (profiling runs)")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 forward leg")
    ap.add_argument("--no-decode", action="store_true", help="skip the decode (split-KV) leg")
    ap.add_argument("--no-workloads", action="store_true", help="skip the gqa / gpt2 / tiny legs")
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(k for k, v in WORKLOADS.items() if not v.nq),
                    help="workload to run (profiling of other shapes; the headline is the default)")
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
