"""Benchmark: SQuad-Attention forward on the Wan-2.2-5B-shaped block (one GPU per rank).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one squad_attn_fwd call (local pass then global pass) over one DiT block's attention:
B=1, h=24, d=128, grid 21x22x40 (n=18480), window 21x2x4 (w=168), bf16, seeded synthetic inputs.
Prints one JSON line (rank 0). With N > 1 (torchrun), every rank runs an independent replica (the
operator has no cross-GPU exchange); timing is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(B=1, h=24, d=128, grid=(21, 22, 40), window=(21, 2, 4), order="local_then_global")
WORKLOAD_NAME = ("Wan-2.2-5B-shaped SQuad attention block: B=1 h=24 d=128, grid 21x22x40 (n=18480), "
                 "window 21x2x4 (w=168, 110 windows), local->global, bf16")
METRIC = "SQuad-attn fwd ms/block & TFLOP/s at n=18480,h=24,d=128 bf16; % of roofline"
PAGES_MS = 4.27   # pages' SQuad attention latency per block for this workload (1x H100, bf16): context
NOMINAL_HBM_GBS = 7700.0   # datasheet HBM3e bandwidth (HGX B200), context beside the measured peak
E2E_GROUPS = 8             # runs of heads of the end-to-end host forward (copies overlap forwards)

# DRAM traffic of one launch of the forward kernel from an ncu capture of this workload
# (dram__bytes_read.sum + dram__bytes_write.sum), valid only for the kernel source it was measured on
# (sha1 prefix below); otherwise reported as null.
PROFILED_TRAFFIC_BYTES = (448.841728 + 192.332288) * 1e6
PROFILED_KERNEL_SHA1 = "d71b1e79836abbc0"
PROFILED_KERNEL_SRC = os.path.join(ROOT, "sub_quadratic_two_squad_b200", "csrc", "attn_short.cu")


def profiled_traffic():
    import hashlib

    try:
        with open(PROFILED_KERNEL_SRC, "rb") as f:
            sha = hashlib.sha1(f.read()).hexdigest()
    except OSError:
        return None
    return PROFILED_TRAFFIC_BYTES if sha.startswith(PROFILED_KERNEL_SHA1) else None


def max_over_ranks(value, world, device=None):
    """Largest `value` over all ranks (device-side timing is reported as the slowest rank)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, "fallback"


def n_tokens(w=WORKLOAD):
    T, H, W = w["grid"]
    return T * H * W


def flops(w=WORKLOAD):
    n = n_tokens(w)
    win = w["window"][0] * w["window"][1] * w["window"][2]
    return 4.0 * w["B"] * w["h"] * w["d"] * (n * win + n * n / win)


def alg_bytes(w=WORKLOAD):
    """Q, K, V read once and O written once (bf16): the roofline's algorithmic traffic of one step."""
    return 4 * w["B"] * w["h"] * n_tokens(w) * w["d"] * 2


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        import torch

        # nvidia-smi numbers GPUs differently from CUDA under CUDA_VISIBLE_DEVICES: address it by UUID.
        try:
            self.dev = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.dev = str(device_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.15)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons), "samples": len(sm)}


def cpu_model():
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def cpu_baseline(budget_s=12.0):
    """The fp64 oracle timed on the host cores, on whole heads of the same workload."""
    import numpy as np
    from threadpoolctl import threadpool_info

    from oracle import squad_oracle as orc
    from sub_quadratic_two_squad_b200.inputs import make_inputs

    w = WORKLOAD
    n = n_tokens(w)
    x = make_inputs(1, 1, n, w["d"], dtype="bf16", heavy_tail=True)
    done, t0 = 0, time.perf_counter()
    while True:
        orc.squad_attn_fwd(x["q"], x["k"], x["v"], w["grid"], w["window"])
        done += 1
        el = time.perf_counter() - t0
        if el >= budget_s or done >= w["h"]:
            break
    per_head_flops = flops(dict(w, h=1))
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    return {"value": per_head_flops * done / el / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"{done} of 24 heads of the same block (fp64 numpy oracle, {el:.1f} s)",
            "ms_per_block_extrapolated": el / done * w["h"] * 1e3}


def run_reference(args, rank, world):
    """--impl reference: the fp64 oracle on the host cores, one bounded sample per step."""
    if rank != 0:
        return
    from threadpoolctl import threadpool_info

    from oracle import squad_oracle as orc
    from sub_quadratic_two_squad_b200.inputs import make_inputs

    w = WORKLOAD
    n = n_tokens(w)
    x = make_inputs(1, 1, n, w["d"], dtype="bf16", heavy_tail=True)
    t0 = time.perf_counter()
    orc.squad_attn_fwd(x["q"], x["k"], x["v"], w["grid"], w["window"])
    t_head = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    heads = max(1, min(w["h"], int(budget / max(t_head, 1e-6))))
    xs = make_inputs(1, heads, n, w["d"], dtype="bf16", heavy_tail=True)
    for _ in range(args.warmup):
        orc.squad_attn_fwd(xs["q"], xs["k"], xs["v"], w["grid"], w["window"])
    t0 = time.perf_counter()
    for _ in range(args.steps):
        orc.squad_attn_fwd(xs["q"], xs["k"], xs["v"], w["grid"], w["window"])
    el = time.perf_counter() - t0
    value = flops(dict(w, h=heads)) * args.steps / el / 1e12
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD_NAME, "sample_heads": heads},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
                             "sample": f"{heads} of 24 heads per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    from sub_quadratic_two_squad_b200 import HostRunner, full_attn_fwd, squad_attn_fwd, squad_attn_fwd_status
    from sub_quadratic_two_squad_b200.inputs import make_inputs

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = WORKLOAD
    n = n_tokens(w)
    shape = (w["B"], w["h"], n, w["d"])
    x = make_inputs(w["B"], w["h"], n, w["d"], dtype="bf16", heavy_tail=True)
    host = {k: torch.from_numpy(v).to(torch.bfloat16) for k, v in x.items()}
    # Rotating buffer sets: each set is 5 x 114 MB (> the 126 MB L2), consecutive steps use different sets.
    n_sets = 3
    sets = []
    for _ in range(n_sets):
        q, k, v = (host[s].to(dev) for s in "qkv")
        o = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        _, ws = squad_attn_fwd(q, k, v, w["grid"], w["window"], w["order"], out=o)
        sets.append((q, k, v, o, ws))
    stream = torch.cuda.current_stream()

    def step(i):
        q, k, v, o, ws = sets[i % n_sets]
        squad_attn_fwd(q, k, v, w["grid"], w["window"], w["order"], out=o, workspace=ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world, dev)
    per_launch_ms = [a.elapsed_time(b) for a, b in ev]
    ms_per_step = total_ms / args.steps
    status_ok = all(squad_attn_fwd_status(s[4], s[0], w["grid"], w["window"], w["order"]) == 0 for s in sets)

    # End to end through the C entry point squad_attn_fwd_host from pinned host buffers: each step copies
    # q, k, v in and o out (inside the timed region), in runs of heads whose copies overlap the forwards.
    runner = HostRunner(w["B"], w["h"], w["d"], w["grid"], w["window"], w["order"], device=dev, groups=E2E_GROUPS)
    hq, hk, hv = (host[s].pin_memory() for s in "qkv")
    ho = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    e2e_steps = max(3, min(args.steps, 30))
    for _ in range(2):
        runner(hq, hk, hv, ho)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    runner.start(a)
    for _ in range(e2e_steps):
        runner(hq, hk, hv, ho)
    runner.end(b)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / e2e_steps, world, dev)

    # Full attention at the same n, beside SQuad (a few calls: ~4.2 TFLOP each).
    q, k, v, o, _ = sets[0]
    full_attn_fwd(q, k, v, grid=w["grid"], out=o)
    torch.cuda.synchronize()
    fa, fb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 5
    fa.record(stream)
    for _ in range(reps):
        full_attn_fwd(q, k, v, grid=w["grid"], out=o)
    fb.record(stream)
    torch.cuda.synchronize()
    full_ms = fa.elapsed_time(fb) / reps
    n_full = 4.0 * w["B"] * w["h"] * w["d"] * n * n

    # Backward at the same shape, beside the forward (a few calls).
    from sub_quadratic_two_squad_b200 import squad_attn_bwd

    q, k, v, o, ws = sets[0]
    dout = torch.from_numpy(make_inputs(w["B"], w["h"], n, w["d"], dtype="bf16", with_dout=True)["do"]).to(dev, torch.bfloat16)
    squad_attn_fwd(q, k, v, w["grid"], w["window"], w["order"], out=o, workspace=ws)
    grads = squad_attn_bwd(q, k, v, o, dout, ws, w["grid"], w["window"], w["order"])
    torch.cuda.synchronize()
    ba, bb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bwd_reps = 20
    ba.record(stream)
    for _ in range(bwd_reps):
        squad_attn_bwd(q, k, v, o, dout, ws, w["grid"], w["window"], w["order"], dq=grads[0], dk=grads[1], dv=grads[2])
    bb.record(stream)
    torch.cuda.synchronize()
    bwd_ms = ba.elapsed_time(bb) / bwd_reps

    # Single-pass variants (one pass alone) at the same shape, rotating the same buffer sets.
    single = {}
    for order in ("local_only", "global_only"):
        q, k, v, o, ws = sets[0]
        squad_attn_fwd(q, k, v, w["grid"], w["window"], order, out=o, workspace=ws)
        torch.cuda.synchronize()
        sa, sb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 30
        sa.record(stream)
        for i in range(reps):
            q, k, v, o, ws = sets[i % len(sets)]
            squad_attn_fwd(q, k, v, w["grid"], w["window"], order, out=o, workspace=ws)
        sb.record(stream)
        torch.cuda.synchronize()
        ms = sa.elapsed_time(sb) / reps
        single[order] = {"ms_per_block": ms, "hbm_frac": alg_bytes() / (ms * 1e-3) / 1e9 / peaks()[0]}

    if rank != 0:
        return
    hbm, tf_peak, peak_kind = peaks()
    f = flops()
    mean_launch = statistics.mean(per_launch_ms)
    achieved = alg_bytes() / (mean_launch * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": world * f / (ms_per_step * 1e-3) / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": PAGES_MS / ms_per_step,
        "vs_baseline_ref": "pages' 4.27 ms per block on 1x H100 80GB bf16 (context, other hardware)",
        "dtype": "bf16",
        "data": "synthetic: seeded N(0,1) Q,K,V rounded to bf16, 2% of key tokens x4 per head",
        "config": {"workload": WORKLOAD_NAME, "global_batch": w["B"], "seq_len": n, "heads": w["h"],
                   "head_dim": w["d"], "window": "21x2x4", "parallelism": f"replicas x{world}" if world > 1 else "1 gpu",
                   "l2": f"{n_sets} rotating buffer sets of ~570 MB each (> 126 MB L2); no reuse between steps"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": profiled_traffic(), "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)",
                     "kernel": "short_kernel (both passes in one launch) + control-block memset",
                     "alg_bytes_per_launch": alg_bytes(), "mean_launch_ms": mean_launch,
                     "tensor_frac": f / (mean_launch * 1e-3) / 1e12 / tf_peak,
                     "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": achieved / NOMINAL_HBM_GBS},
        "e2e": {"value": world * f / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": runner.h2d_bytes(), "d2h_bytes_per_step": runner.d2h_bytes(),
                "steps": e2e_steps, "groups": E2E_GROUPS,
                "api": "C entry point squad_attn_fwd_host (pinned host buffers, runs of heads on three streams)"},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "device_status_ok": status_ok,
        "full_attn": {"ms_per_block": full_ms, "tflops": n_full / (full_ms * 1e-3) / 1e12,
                      "flop_ratio": n_full / f, "latency_ratio": full_ms / ms_per_step},
        "single_pass": single,
        "backward": {"ms_per_block": bwd_ms,
                     "tflops_algorithmic": 2.0 * f / (bwd_ms * 1e-3) / 1e12,
                     "flops_note": "algorithmic = 2x forward (dQ, dK, dV, dP products); executed: 2.5x forward "
                                   "(S and dP once; the 168-token windows' P and dS pass through an L2 scratch "
                                   "to the column products, the 110-token slot sequences through shared memory)",
                     "kernels": "tcgen05, one persistent launch per pass (one CTA per SM; row-owner, epilogue "
                                "and load/MMA warps): bwd_tc1_kernel (slot sequences) then bwd_tc_kernel (windows)"},
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


# Every block shape the measurements cover (name, B, h, d, grid, window, orders, with full attention,
# with backward). Timed by `--sweep`, one JSON line each; the default run times only the 5B block.
SWEEP = [
    ("Wan-2.2-5B block", 1, 24, 128, (21, 22, 40), (21, 2, 4),
     ("local_then_global", "global_then_local", "local_only", "global_only"), True, True),
    ("Wan-2.1-1.3B block", 1, 12, 128, (21, 30, 52), (21, 2, 4), ("local_then_global", "global_then_local"), False, False),
    ("high-resolution 5B block", 1, 24, 128, (21, 44, 80), (21, 4, 4), ("local_then_global", "local_only", "global_only"),
     True, True),
    ("Wan-2.1-14B block (training step)", 1, 40, 128, (21, 22, 40), (21, 2, 4), ("local_then_global",), False, True),
    ("Wan-2.2-5B grid, window 21x3x4 (reflect-padded to 21x24x40)", 1, 24, 128, (21, 22, 40), (21, 3, 4),
     ("local_then_global",), False, True),
]

# k composed passes over nested windows on the Wan-2.2-5B grid: (name, B, h, d, grid, levels, orders, with_bwd).
KPASS_SWEEP = [
    ("Wan-2.2-5B block, k = 3 (levels 1x1, 11x2, 2x20: 21 + 22 + 40 tokens)", 1, 24, 128, (21, 22, 40),
     [(1, 1), (11, 2), (2, 20)], ("forward", "reverse"), True),
    ("Wan-2.2-5B block, k = 3 (levels 2x4, 11x2, 1x5: 168 + 22 + 5 tokens)", 1, 24, 128, (21, 22, 40),
     [(2, 4), (11, 2), (1, 5)], ("forward",), False),
]


def sweep(reps=30, only=None, n_sets=3):
    """Forward (and backward, full attention) device times for every block shape, N(0,1) inputs drawn on
    the device, 3 rotating buffer sets, CUDA events on the launching stream."""
    import torch

    from sub_quadratic_two_squad_b200 import (full_attn_fwd, squad_attn_bwd, squad_attn_bwd_kernels, squad_attn_flops,
                                              squad_attn_fwd)

    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    hbm, tf_peak, peak_kind = peaks()

    def timed(fn, n_rep):
        fn(0)
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(n_rep):
            fn(i)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n_rep

    for name, B, h, d, grid, window, orders, with_full, with_bwd in SWEEP:
        if only is not None and only not in name:
            continue
        w = dict(B=B, h=h, d=d, grid=grid, window=window)
        n = n_tokens(w)
        ns = n_sets
        sets = [tuple(torch.randn(B, h, n, d, device=dev, dtype=torch.bfloat16) for _ in range(3)) for _ in range(ns)]
        outs = [torch.empty_like(x[0]) for x in sets]
        for order in orders:
            wss = [squad_attn_fwd(*sets[i], grid, window, order)[1] for i in range(ns)]
            ms = timed(lambda i: squad_attn_fwd(*sets[i % ns], grid, window, order, out=outs[i % ns],
                                                workspace=wss[i % ns]), reps)
            f = squad_attn_flops(B, h, d, grid, window, order)   # the padded grid's cost where it pads
            t_roof = max(f / (tf_peak * 1e12), alg_bytes(w) / (hbm * 1e9)) * 1e3
            line = {"sweep": name, "order": order, "n": n, "window": "x".join(map(str, window)), "ms_per_block": ms,
                    "tflops": f / (ms * 1e-3) / 1e12, "roofline_ms": t_roof, "roofline_frac": t_roof / ms,
                    "hbm_gbs_algorithmic": alg_bytes(w) / (ms * 1e-3) / 1e9, "peaks": peak_kind}
            if with_bwd and order == "local_then_global":
                dout = torch.randn(B, h, n, d, device=dev, dtype=torch.bfloat16)
                q, k, v = sets[0]
                o, ws = squad_attn_fwd(q, k, v, grid, window, order)
                g = squad_attn_bwd(q, k, v, o, dout, ws, grid, window, order)
                bms = timed(lambda i: squad_attn_bwd(q, k, v, o, dout, ws, grid, window, order, dq=g[0], dk=g[1],
                                                     dv=g[2]), 10)
                bwd_bytes = 8 * B * h * n * d * 2   # Q, K, V, O, dO in; dQ, dK, dV out (bf16), + O1 once
                line["backward"] = {"ms_per_block": bms, "tflops_algorithmic": 2 * f / (bms * 1e-3) / 1e12,
                                    "hbm_frac_8_tensors": bwd_bytes / (bms * 1e-3) / 1e9 / hbm,
                                    "kernels": squad_attn_bwd_kernels(B, h, d, grid, window, order)}
            print(json.dumps(line), flush=True)
            del wss
        if with_full:
            q, k, v = sets[0]
            fms = timed(lambda i: full_attn_fwd(*sets[i % ns], grid=grid, out=outs[i % ns]), 3)
            nf = 4.0 * B * h * d * n * n
            print(json.dumps({"sweep": name, "order": "full_attn_fwd", "n": n, "ms_per_block": fms,
                              "tflops": nf / (fms * 1e-3) / 1e12, "tensor_frac": nf / (fms * 1e-3) / 1e12 / tf_peak}),
                  flush=True)
        del sets, outs
        torch.cuda.empty_cache()

    from sub_quadratic_two_squad_b200 import squad_kpass_bwd, squad_kpass_flops, squad_kpass_fwd

    for name, B, h, d, grid, levels, orders, with_bwd in KPASS_SWEEP:
        if only is not None and only not in name:
            continue
        w = dict(B=B, h=h, d=d, grid=grid, window=(grid[0], 1, 1))
        n = n_tokens(w)
        ns = n_sets
        sets = [tuple(torch.randn(B, h, n, d, device=dev, dtype=torch.bfloat16) for _ in range(3)) for _ in range(ns)]
        outs = [torch.empty_like(x[0]) for x in sets]
        f = squad_kpass_flops(B, h, d, grid, levels)
        for order in orders:
            wss = [squad_kpass_fwd(*sets[i], grid, levels, order)[1] for i in range(ns)]
            ms = timed(lambda i: squad_kpass_fwd(*sets[i % ns], grid, levels, order, out=outs[i % ns],
                                                 workspace=wss[i % ns]), reps)
            t_roof = max(f / (tf_peak * 1e12), alg_bytes(w) / (hbm * 1e9)) * 1e3
            line = {"sweep": name, "order": order, "n": n, "levels": ["x".join(map(str, l)) for l in levels],
                    "ms_per_block": ms, "tflops": f / (ms * 1e-3) / 1e12, "roofline_ms": t_roof,
                    "roofline_frac": t_roof / ms, "hbm_gbs_algorithmic": alg_bytes(w) / (ms * 1e-3) / 1e9,
                    "peaks": peak_kind}
            if with_bwd and order == "forward":
                dout = torch.randn(B, h, n, d, device=dev, dtype=torch.bfloat16)
                q, k, v = sets[0]
                o, ws = squad_kpass_fwd(q, k, v, grid, levels, order)
                g = squad_kpass_bwd(q, k, v, o, dout, ws, grid, levels, order)
                bms = timed(lambda i: squad_kpass_bwd(q, k, v, o, dout, ws, grid, levels, order, dq=g[0], dk=g[1],
                                                      dv=g[2]), 10)
                line["backward"] = {"ms_per_block": bms, "tflops_algorithmic": 2 * f / (bms * 1e-3) / 1e12}
            print(json.dumps(line), flush=True)
            del wss
        del sets, outs
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="time every block shape (one JSON line each) and exit")
    ap.add_argument("--only", default=None, help="with --sweep: only the block shapes whose name contains this")
    ap.add_argument("--sets", type=int, default=3, help="with --sweep: rotating buffer sets (3 keep inputs > L2)")
    ap.add_argument("--reps", type=int, default=30, help="with --sweep: timed calls per order")
    args = ap.parse_args()
    if args.sweep:
        sweep(reps=args.reps, only=args.only, n_sets=args.sets)
        return
    args.warmup = max(args.warmup, 3)
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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local_rank))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
