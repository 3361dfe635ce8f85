#!/usr/bin/env python
"""Benchmark of the Muon / Aurora optimizer step on B200.

One step = one full optimizer step (momentum + Nesterov, power iteration,
Aurora-equilibrated Newton-Schulz polar, contra subtraction and Frobenius
restore, aspect scale, u/w floor, parameter add) over every 2-D matrix of the
workload, through the library's C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (the float64 CPU oracle, same metric)

Default workload: the 3.8B Llama-style matrix set (28 layers, 168 matrices,
2.82 G parameters) with the full Aurora + Contra-Muon + u/w-floor stack,
bf16 params/grads, fp32 momentum.  Inputs are synthetic (seeded) and larger
than L2, so no flush is needed between steps.  For N > 1 (torchrun) the
matrices are sharded by LPT over ranks and one NCCL all-gather of the
updated parameters closes each step (strong scaling).  Rank 0 prints one
JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = "Muon/Aurora steps/s & NS TFLOP/s (% bf16 peak) on 3.8B matrix shapes"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama_aurora", choices=sorted(WL.WORKLOADS) + ["llama_aux"])
    ap.add_argument("--layers", type=int, default=28, help="layers of the 3.8B set (28 = full)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm", default="bf16", choices=["bf16", "fp32", "bf16simt"])
    ap.add_argument("--graph", action="store_true",
                    help="one GPU: capture the step in a CUDA graph and time its replays (for launch-bound "
                         "workloads); the per-stage figures then come from one eager step after the timed region")
    ap.add_argument("--ns-vs-cublas", action="store_true",
                    help="time one Newton-Schulz polar of the workload's matrices on this library (ns_polar) "
                         "and the same iteration on torch/cuBLAS bf16 bmm, alternating; prints one JSON line")
    return ap.parse_args()


AUX_WORKLOADS = {"llama_aux": WL.llama_3p8b_aux}
AUX_METRIC = "AdamW auxiliary-parameter steps/s on the 3.8B non-matrix set (GB/s, % of HBM)"


def make_workload(args):
    if args.workload in AUX_WORKLOADS:
        return AUX_WORKLOADS[args.workload](layers=args.layers)
    if args.workload in ("llama_plain", "llama_aurora"):
        return WL.WORKLOADS[args.workload](layers=args.layers)
    return WL.WORKLOADS[args.workload]()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def nominal_ns_flops(wl) -> float:
    c = wl.cfg
    tot = 0.0
    for m, n in wl.shapes:
        s, l = min(m, n), max(m, n)
        polars = c.pp_iterations if (c.aurora and m != n) else 1
        tot += polars * c.ns_steps * (4.0 * s * s * l + 2.0 * s ** 3)
    return tot


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
            return
        # the first reading lands before the timed region starts, so a region
        # shorter than the sampling period still carries one
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5.0 and self.proc.poll() is None:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------- CPU oracle leg
def oracle_sample_time(wl, indices):
    """Wall time of the float64 oracle stepping `indices` of the workload once."""
    import oracle.muon_oracle as O
    Ws, Gs, Ms = WL.generate(wl, indices)
    t0 = time.perf_counter()
    for k, i in enumerate(indices):
        O.step(WL.to_f64(Ws[k], wl.param_dtype), WL.to_f64(Gs[k], wl.grad_dtype), Ms[k].astype(np.float64),
               wl.cfg, wl.param_dtype)
    return time.perf_counter() - t0


def sample_plan(wl):
    """Matrices the oracle steps for the CPU figures, and how many matrices of
    the workload each one stands for.

    The layered sets (the 3.8B model, GPT-2) time all six matrices of layer 0
    (q, k, v, o, fc, proj) and scale by the layer count: every layer has the
    same shapes, and the oracle's cost depends only on the shapes.  The
    Aurora sweep times one matrix of each shape and weights it by that
    shape's count; small sets are timed whole."""
    if wl.name.startswith("llama") or wl.name.startswith("gpt2"):
        per_layer = 6
        layers = wl.n // per_layer
        assert layers * per_layer == wl.n and wl.shapes == wl.shapes[:per_layer] * layers
        return list(range(per_layer)), [layers] * per_layer
    if wl.n <= 8:
        return list(range(wl.n)), [1] * wl.n
    first, count = {}, {}
    for i, shp in enumerate(wl.shapes):
        first.setdefault(shp, i)
        count[shp] = count.get(shp, 0) + 1
    idx = sorted(first.values())
    return idx, [count[wl.shapes[i]] for i in idx]


def _sample_desc(wl, idx, weights):
    names = ",".join(f"{wl.shapes[i][0]}x{wl.shapes[i][1]}" for i in idx)
    scale = weights[0] if len(set(weights)) == 1 else weights
    return names, scale


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([d.get("num_threads", 1) for d in info] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl):
    """The oracle steps each sampled matrix once; the step time is the sum of
    their times, each multiplied by the number of matrices it stands for."""
    idx, weights = sample_plan(wl)
    ts = [oracle_sample_time(wl, [i]) for i in idx]
    step_s = sum(w * t for w, t in zip(weights, ts))
    names, scale = _sample_desc(wl, idx, weights)
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
            "extrapolated": len(idx) < wl.n, "timed_matrices": len(idx), "scale": scale,
            "sample_wall_s": sum(ts),
            "sample": f"{len(idx)} of {wl.n} matrices ({names}) stepped once each by the float64 NumPy oracle "
                      f"in {sum(ts):.1f} s; step time = sum of their times x the matrices each stands for "
                      f"({scale})"}


def run_reference(args):
    """The oracle on the host cores, on the same workload, metric and unit.

    Each timed step runs the oracle on one sampled matrix in turn (more than
    one when there are fewer steps than sampled matrices), so every sampled
    matrix is timed at least once and the whole run stays within minutes; the
    reported step time is the sum over the sample of each matrix's mean time
    times the matrices it stands for.  A warm-up step runs the oracle once on
    the smallest sampled matrix (the oracle has no state to warm up; this
    only starts the BLAS thread pool)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = make_workload(args)
    idx, weights = sample_plan(wl)
    smallest = min(idx, key=lambda i: wl.shapes[i][0] * wl.shapes[i][1])
    for _ in range(args.warmup):
        oracle_sample_time(wl, [smallest])
    steps = max(1, args.steps)
    times = {i: [] for i in idx}
    total = max(steps, len(idx))
    for j in range(total):
        i = idx[j % len(idx)]
        times[i].append(oracle_sample_time(wl, [i]))
    step_s = sum(w * (sum(times[i]) / len(times[i])) for i, w in zip(idx, weights))
    v = 1.0 / step_s
    names, scale = _sample_desc(wl, idx, weights)
    wall = sum(sum(t) for t in times.values())
    sample = (f"each step: the float64 oracle on one of {len(idx)} of {wl.n} matrices ({names}) in turn; step time "
              f"= sum of each sampled matrix's mean time x the matrices it stands for ({scale}); {wall:.1f} s of "
              f"oracle time over {steps} steps; warm-up: the oracle once on the smallest sampled matrix")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "matrices": wl.n, "elements": wl.elements()},
        "extrapolated": len(idx) < wl.n,
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                         "extrapolated": len(idx) < wl.n, "timed_matrices": len(idx), "scale": scale,
                         "sample_wall_s": wall, "sample": sample},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- AdamW leg
AUX_BYTES_PER_ELEM = {("bf16", "bf16"): 2 + 2 + 2 + 8 + 8, ("f32", "f32"): 4 + 4 + 4 + 8 + 8}


def aux_oracle_time(wl, idx):
    import oracle.muon_oracle as O
    P = [WL.aux_param(wl, i) for i in idx]
    G = [WL.aux_grad(wl, i, 1) for i in idx]
    t0 = time.perf_counter()
    for k, i in enumerate(idx):
        z = np.zeros(wl.shapes[i])
        O.adamw_step(WL.to_f64(P[k], wl.param_dtype), WL.to_f64(G[k], wl.grad_dtype), z, z, wl.lrs[i], wl.beta1,
                     wl.beta2, wl.eps, wl.weight_decay, 1)
    return time.perf_counter() - t0


def aux_cpu_line(wl, reps):
    idx = [2] + list(range(16, min(wl.n, 24)))          # one value-embedding table and some 1-D tensors
    elems = sum(int(np.prod(wl.shapes[i])) for i in idx)
    ts = [aux_oracle_time(wl, idx) for _ in range(reps)]
    step_s = sum(ts) / len(ts) * wl.elements() / elems
    return 1.0 / step_s, {"value": 1.0 / step_s, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                          "sample": f"{len(idx)} of {wl.n} tensors ({elems / 1e6:.1f} M elements) stepped by the "
                                    f"float64 NumPy oracle, scaled by element count (x{wl.elements() / elems:.1f})"}


def run_aux(args, wl):
    import torch
    from aurora_orthogonalised_optimizer_b200 import _abi as A
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        raise SystemExit("the AdamW workload runs on one GPU")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    pdt = torch.bfloat16 if wl.param_dtype == WL.BF16 else torch.float32

    def dev_tensor(a, dt):
        if dt == WL.BF16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    p = [dev_tensor(WL.aux_param(wl, i), wl.param_dtype) for i in range(wl.n)]
    g = [dev_tensor(WL.aux_grad(wl, i, 1), wl.grad_dtype) for i in range(wl.n)]
    m = [torch.zeros(s, dtype=torch.float32, device=dev) for s in wl.shapes]
    v = [torch.zeros(s, dtype=torch.float32, device=dev) for s in wl.shapes]
    stream = torch.cuda.current_stream(dev)
    step_no = [0]

    def step():
        step_no[0] += 1
        A.adamw_step(p, g, m, v, step_no[0], wl.lrs, wl.beta1, wl.beta2, wl.eps, wl.weight_decay, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = "0"
    clocks = ClockSampler(gpu_id)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    launches_per_step = (wl.n + 191) // 192
    bytes_step = wl.elements() * AUX_BYTES_PER_ELEM[(wl.param_dtype, wl.grad_dtype)]
    peaks, kind = load_peaks()
    hbm = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    gbs = bytes_step / ms / 1e6
    e2e = None
    if not args.no_e2e:
        g_pin = [t.cpu().pin_memory() for t in g]
        p_pin = [torch.empty_like(t, device="cpu").pin_memory() for t in p]
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(args.steps):
            for k in range(wl.n):
                g[k].copy_(g_pin[k], non_blocking=True)
            step()
            for k in range(wl.n):
                p_pin[k].copy_(p[k], non_blocking=True)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e = {"value": 1e3 * args.steps / f0.elapsed_time(f1), "unit": "steps/s",
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in g_pin),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in p_pin)}
    cpu = None
    if not args.no_cpu_baseline:
        _, cpu = aux_cpu_line(wl, 1)
    line = {
        "metric": AUX_METRIC, "value": 1e3 / ms, "unit": "steps/s", "n_gpus": 1, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0, 0.02^2) params, N(0, 1e-6) grads)",
        "config": {"workload": wl.name, "tensors": wl.n, "elements": wl.elements(),
                   "l2": (f"{bytes_step / 1e9:.1f} GB of operands per step, larger than the 126 MB L2; no flush"
                          if bytes_step > 126e6 else f"{bytes_step / 1e6:.1f} MB of operands per step fit in the "
                          "126 MB L2; no flush (a launch-bound case)")},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                     "traffic": None, "kernel": "k_adamw", "peak_kind": f"hbm_gbs ({kind})",
                     "bytes_per_launch": bytes_step / launches_per_step},
        "gpu_launches": launches_per_step * args.steps, "clocks": clk, "e2e": e2e, "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU leg
def run_ns_vs_cublas(args):
    """Context measurement: the same Newton-Schulz polar (ns_steps x {A = X X^T,
    B = b A + c A^2, X = a X + B X} over every matrix of the workload, bf16
    operands) through ns_polar and through torch.bmm/baddbmm on cuBLAS, in
    alternating rounds on the same GPU with clocks sampled.  FLOPs are counted
    the library's way (one triangle of each symmetric product) for both."""
    import torch
    from aurora_orthogonalised_optimizer_b200 import _abi as A
    wl = make_workload(args)
    dev = torch.cuda.current_device()
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    c = wl.cfg
    buckets = {}
    for m, n in wl.shapes:
        key = (min(m, n), max(m, n))
        buckets[key] = buckets.get(key, 0) + 1
    useful = sum(cnt * c.ns_steps * (l * s * (s + 1) + s * s * (s + 1) + 2.0 * s * s * l)
                 for (s, l), cnt in buckets.items())
    g = torch.Generator(device="cuda").manual_seed(0)
    X = {k: torch.randn(cnt, k[0], k[1], device="cuda", dtype=torch.bfloat16, generator=g) / (k[0] * k[1]) ** 0.5
         for k, cnt in buckets.items()}
    ins = [torch.randn(m, n, device="cuda", dtype=torch.bfloat16, generator=g) for m, n in wl.shapes]
    outs = [torch.empty(m, n, device="cuda", dtype=torch.float32) for m, n in wl.shapes]
    cfg = A.Config.from_step_config(c, gemm_mode=A.MUON_GEMM_BF16)
    ws = A.make_workspace(cfg, wl.shapes)

    def cublas_polar():
        for x in X.values():
            for _ in range(c.ns_steps):
                a = torch.bmm(x, x.transpose(1, 2))
                b = torch.baddbmm(a, a, a, beta=c.ns_b, alpha=c.ns_c)
                x = torch.baddbmm(x, b, x, beta=c.ns_a, alpha=1.0)

    def ours():
        A.ns_polar(cfg, ins, outs, ws)

    def timed(fn, reps):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    for _ in range(max(1, args.warmup)):
        ours()
        cublas_polar()
    rows = {"library_ns_polar": [], "cublas_bmm": []}
    for _ in range(max(1, args.steps)):
        for name, fn in (("library_ns_polar", ours), ("cublas_bmm", cublas_polar)):
            cs = ClockSampler(gpu_id)
            cs.start()
            if name == "library_ns_polar":
                A.profile_enable(True)
            ms = timed(fn, 3)
            row = {"ms_per_polar": ms, "useful_tflops": useful / ms / 1e9}
            if name == "library_ns_polar":
                prof = A.profile_read()
                A.profile_enable(False)
                gm = prof.get("ns_gemm_tc")
                if gm:
                    row["gemm_ms_per_polar"] = gm["ms"] / 3
                    row["gemm_useful_tflops"] = gm["flops"] / gm["ms"] / 1e9
            row["clocks"] = cs.stop()
            rows[name].append(row)
    best = {k: min(v, key=lambda r: r["ms_per_polar"]) for k, v in rows.items()}
    print(json.dumps({"metric": "Newton-Schulz polar of the workload's matrices, library vs torch/cuBLAS",
                      "workload": wl.name, "ns_steps": c.ns_steps, "useful_gflop_per_polar": useful / 1e9,
                      "library": best["library_ns_polar"], "cublas": best["cublas_bmm"],
                      "speedup": best["cublas_bmm"]["ms_per_polar"] / best["library_ns_polar"]["ms_per_polar"],
                      "rounds": rows}), flush=True)
    return 0


def traffic_record(kernel_src):
    """Per-launch DRAM traffic from the committed ncu summary, if taken on this exact kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        d = json.load(open(p))
        h = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
        if d.get("source_sha256_16") != h:
            return None
        return d
    except Exception:
        return None


def main():
    args = parse()
    if args.ns_vs_cublas:
        return run_ns_vs_cublas(args)
    if args.workload in AUX_WORKLOADS:
        if args.impl == "reference":
            if int(os.environ.get("RANK", "0")) != 0:
                return 0
            wl = make_workload(args)
            for _ in range(args.warmup):
                aux_cpu_line(wl, 1)
            v, cpu = aux_cpu_line(wl, args.steps)
            print(json.dumps({"impl": "reference", "metric": AUX_METRIC, "value": v, "unit": "steps/s",
                              "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": 1e3 / v, "higher_is_better": True, "scaling": "strong",
                              "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                              "config": {"workload": wl.name}, "cpu_baseline": cpu,
                              "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0,
                                      "d2h_bytes_per_step": 0}}), flush=True)
            return 0
        return run_aux(args, make_workload(args))
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    from aurora_orthogonalised_optimizer_b200 import _abi as A
    from aurora_orthogonalised_optimizer_b200 import sharding as SH

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    wl = make_workload(args)
    gemm = {"bf16": A.MUON_GEMM_BF16, "fp32": A.MUON_GEMM_FP32, "bf16simt": A.MUON_GEMM_BF16_SIMT}[args.gemm]
    cfg = A.Config.from_step_config(wl.cfg, gemm_mode=gemm,
                                    param_dtype=1 if wl.param_dtype == WL.BF16 else 0,
                                    grad_dtype=1 if wl.grad_dtype == WL.BF16 else 0)
    shapes = wl.shapes
    costs = SH.step_costs(shapes, wl.cfg.ns_steps, wl.cfg.aurora, wl.cfg.pp_iterations)
    owned_all = SH.lpt_partition(costs, world)
    owned = owned_all[rank]
    layout = SH.flat_layout(shapes, owned_all)
    pdt = torch.bfloat16 if wl.param_dtype == WL.BF16 else torch.float32
    gdt = torch.bfloat16 if wl.grad_dtype == WL.BF16 else torch.float32

    # ---- inputs: every rank holds all params (flat, sharded layout); grads and momentum of its own matrices
    threads = min(32, os.cpu_count() or 8)
    flat = torch.empty(layout.total_elems, dtype=pdt, device=dev)
    pviews = SH.views(flat, layout, shapes)
    W_host, G_host = WL.generate_torch(wl, owned, 0, threads)
    for k, i in enumerate(owned):
        pviews[i].copy_(W_host[k])
    if world > 1:
        SH.exchange(flat, layout, rank)
    params = [pviews[i] for i in owned]
    grads = [G_host[k].to(dev) for k in range(len(owned))]
    mom = [torch.zeros(shapes[i], dtype=torch.float32, device=dev) for i in owned]
    my_shapes = [shapes[i] for i in owned]
    ws = A.make_workspace(cfg, my_shapes, dev)
    del W_host
    stream = torch.cuda.current_stream(dev)

    def step():
        A.muon_step(cfg, params, grads, mom, None, ws, stream)
        if world > 1:
            SH.exchange(flat, layout, rank)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    if A.last_device_status(stream) != A.MUON_OK:
        raise SystemExit("device status error during warm-up")
    graph = None
    if args.graph:
        if world > 1:
            raise SystemExit("--graph is for one GPU")
        # the step issues only kernel launches and workspace memsets on its stream: capture one and replay it
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            A.muon_step(cfg, params, grads, mom, None, ws)
        torch.cuda.synchronize()
        graph.replay()
        torch.cuda.synchronize()
        eager_step = step

        def step():
            graph.replay()

    # ---- timed region (device time, CUDA events on the launch stream)
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        gpu_id = str(local)
    clocks = ClockSampler(gpu_id)
    A.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    A.profile_enable(False)
    prof = A.profile_read()
    ms = e0.elapsed_time(e1)
    if graph is not None:
        # replays record no per-launch events: take the stage split from one eager step
        A.profile_enable(True)
        eager_step()
        torch.cuda.synchronize()
        A.profile_enable(False)
        prof = A.profile_read()
        for v in prof.values():
            for k in ("launches", "ms", "flops", "bytes"):
                v[k] = v[k] * args.steps
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps
    steps_per_s = 1e3 / ms_per_step

    # ---- end to end: grads host->device from pinned memory, step, params device->host.
    # Every step's grads are copied in and its updated params copied out
    # inside the timed region, pipelined the way a training loop would run it:
    # the next step's grads go into a second device buffer on an input copy
    # stream while this step computes, and the updated params are snapshotted
    # on the device (one device-to-device copy) and read back on an output
    # copy stream while the next step runs.  The region ends after the last
    # read-back has landed in host memory.
    e2e = None
    if not args.no_e2e:
        g_pin = [G_host[k].pin_memory() for k in range(len(owned))]
        p_pin = [torch.empty(shapes[i], dtype=pdt).pin_memory() for i in owned]
        h2d = sum(t.numel() * t.element_size() for t in g_pin)
        d2h = sum(t.numel() * t.element_size() for t in p_pin)
        gbuf = [grads, [torch.empty_like(g) for g in grads]]
        snap = [torch.empty_like(q) for q in params]
        cs_in = torch.cuda.Stream(device=dev)
        cs_out = torch.cuda.Stream(device=dev)
        h2d_done = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]
        snap_ready, snap_free = torch.cuda.Event(), torch.cuda.Event()
        barrier()
        torch.cuda.synchronize()
        f0 = torch.cuda.Event(enable_timing=True)
        f1 = torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        cs_in.wait_event(f0)

        def copy_in(b):
            with torch.cuda.stream(cs_in):
                for k in range(len(owned)):
                    gbuf[b][k].copy_(g_pin[k], non_blocking=True)
                h2d_done[b].record(cs_in)

        copy_in(0)
        for s_ in range(args.steps):
            b = s_ % 2
            if s_ + 1 < args.steps:
                if s_ >= 1:
                    cs_in.wait_event(used[1 - b])      # step s_-1 has consumed that buffer
                copy_in(1 - b)
            stream.wait_event(h2d_done[b])
            A.muon_step(cfg, params, gbuf[b], mom, None, ws, stream)
            if world > 1:
                SH.exchange(flat, layout, rank)
            used[b].record(stream)
            if s_ >= 1:
                stream.wait_event(snap_free)           # the previous read-back is done with snap
            for k in range(len(owned)):
                snap[k].copy_(params[k], non_blocking=True)
            snap_ready.record(stream)
            cs_out.wait_event(snap_ready)
            with torch.cuda.stream(cs_out):
                for k in range(len(owned)):
                    p_pin[k].copy_(snap[k], non_blocking=True)
                snap_free.record(cs_out)
        stream.wait_event(snap_free)
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ems = f0.elapsed_time(f1)
        if world > 1:
            t = torch.tensor([ems], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ems = float(t.item())
        e2e = {"value": 1e3 * args.steps / ems, "unit": "steps/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h,
               "copies": "every step's grads in and params out, overlapped with compute on two copy streams "
                         "(double-buffered grads, device snapshot of the params)"}
        if world > 1:
            tot = torch.tensor([h2d, d2h], dtype=torch.float64, device=dev)
            dist.all_reduce(tot)
            e2e["h2d_bytes_per_step"], e2e["d2h_bytes_per_step"] = int(tot[0].item()), int(tot[1].item())

    if A.last_device_status(stream) != A.MUON_OK:
        raise SystemExit("device status error in the timed region")

    # ---- roofline of the dominant kernel + per-stage figures
    peaks, peak_kind = load_peaks()
    gk = "ns_gemm_tc" if gemm == A.MUON_GEMM_BF16 else "ns_gemm_simt"
    g = prof.get(gk, {"launches": 0, "ms": 0.0, "flops": 0.0})
    kinds = {k[len("tc_kind_"):]: v for k, v in prof.items() if k.startswith("tc_kind_")}
    prof = {k: v for k, v in prof.items() if not k.startswith("tc_kind_")}
    launches = sum(v["launches"] for v in prof.values())
    achieved_tf = g["flops"] / max(g["ms"], 1e-9) / 1e9  # flops / ms -> TFLOP/s
    traffic = None
    if gk == "ns_gemm_tc":
        bound = "tensor"
        peak_tf = peaks.get("bf16_tflops_sustained", PEAKS_FALLBACK["bf16_tflops_sustained"])
        peak_desc = f"bf16_tflops_sustained ({peak_kind})"
        tr = traffic_record(os.path.join(ROOT, "aurora_orthogonalised_optimizer_b200", "csrc", "gemm_tc.cu"))
        if tr is not None and g["launches"]:
            traffic = tr.get("bytes_per_flop", 0.0) * g["flops"] / g["launches"]
    else:
        # fp32 FMA on the CUDA cores: 128 fp32 lanes per SM, 2 FLOP per FMA, at
        # the highest SM clock the sampler saw
        bound = "alu"
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = (clk or {}).get("sm_max_mhz") or 1965.0
        peak_tf = sms * 128 * 2 * mhz * 1e6 / 1e12
        peak_desc = f"fp32 FMA, derived: {sms} SMs x 128 lanes x 2 FLOP x {mhz:.0f} MHz"
    roofline = {"bound": bound, "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved_tf / peak_tf, "traffic": traffic,
                "kernel": "k_gemm_tc" if gk == "ns_gemm_tc" else "k_gemm_simt",
                "peak_kind": peak_desc,
                "flops_per_launch": g["flops"] / max(1, g["launches"]),
                "ms_per_launch": g["ms"] / max(1, g["launches"])}
    hbm = peaks.get("hbm_gbs", PEAKS_FALLBACK["hbm_gbs"])
    stages = {}
    for k, v in prof.items():
        if v["launches"] == 0:
            continue
        st = {"launches": v["launches"] // args.steps, "ms_per_step": v["ms"] / args.steps,
              "share": v["ms"] / max(sum(x["ms"] for x in prof.values()), 1e-9)}
        if v["bytes"] > 0:
            st["GB/s"] = v["bytes"] / v["ms"] / 1e6
            st["frac_hbm"] = st["GB/s"] / hbm
        if v["flops"] > 0:
            st["TFLOP/s"] = v["flops"] / v["ms"] / 1e9
        stages[k] = st
    if gk in stages and kinds:
        # the tensor-core GEMM launches split by kind (Gram, square, update)
        stages[gk]["kinds"] = {k: {"launches": v["launches"] // args.steps, "ms_per_step": v["ms"] / args.steps,
                                   "TFLOP/s": v["flops"] / max(v["ms"], 1e-9) / 1e9}
                               for k, v in kinds.items() if v["launches"]}
    ns_nominal = nominal_ns_flops(wl)
    ns_tf_nominal = ns_nominal * steps_per_s / 1e12

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        # bytes a step reads at least once: params, grads, fp32 momentum
        in_gb = wl.elements() * ((2 if pdt == torch.bfloat16 else 4) + (2 if gdt == torch.bfloat16 else 4) + 4) / 1e9
        l2_note = (f"inputs ({in_gb:.1f} GB) larger than the 126 MB L2; no flush" if in_gb > 0.126 else
                   f"inputs ({1e3 * in_gb:.1f} MB) fit in the 126 MB L2; no flush (a launch-bound case)")
        line = {
            "metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16" if gemm != A.MUON_GEMM_FP32 else "f32",
            "data": "synthetic (seeded N(0,1) grads x 1e-3 with log-normal(0,0.5) row scales, N(0,1/fan_in) "
                    "weights)" if wl.name.startswith("llama") else "synthetic (seeded)",
            "config": {"workload": wl.name, "matrices": wl.n, "elements": wl.elements(),
                       "parallelism": f"matrix-sharded x{world} (LPT) + all-gather" if world > 1 else "single GPU",
                       "gemm": args.gemm, "l2": l2_note},
            "matrices_per_s": wl.n * steps_per_s,
            "ns_tflops_dense_equivalent": ns_tf_nominal,
            "roofline": roofline,
            "stages": stages,
            "gpu_launches": launches,
            "clocks": clk,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
