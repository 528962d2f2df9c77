#!/usr/bin/env python
"""Benchmark of the AWQ W4A16 g128 hot path on B200.

Headline (the default workload, Llama-2-7B decode at M = 1): effective weight
GB/s of the decode GEMV. One step is one decode pass over the four linear
layers of a Llama-2-7B block (4096x12288 qkv, 4096x4096 o_proj, 4096x22016
gate+up, 11008x4096 down): four awq_w4a16_gemv launches on weights that were
folded and quantized once before the timed region (as a deployed model's
are) and are rotated over enough packed copies (>= 4x the L2 size) that every
step streams them from HBM. value = fp16-equivalent weight bytes (2 per
weight) per second.

Sub-records in the same JSON line, each with its own roofline:
  gemv_layers   every decode layer alone (C2 and the two Llama-2-70B layers, M = 1)
  gemm          the prefill GEMM on Llama-3-8B gate+up (4096x28672) at M = 4096, TFLOP/s
  quantize      the fold + quantizer over each full Llama-2-70B layer, GB/s
  act_scale     the activation statistic + scaling at 4096 x 4096, GB/s
  full_path     one pass of every row of the path (a1 + a2 + a3 per layer) on the default workload
  decode_layer_chain  one Llama-2-7B block's linear layers at M = 1 as a dependent chain (scaling,
                fused q/k/v, o_proj, fused gate/up SiLU*up, down) in a CUDA graph

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME] [--m M]

Under torchrun each rank runs its own replica (weak scaling, no data-path
collective); timing is on the device with CUDA events, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

GROUP = 128
L2_BYTES_DEFAULT = 126 * 1024 * 1024


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama2_7b_decode_m1", choices=workloads.workload_names())
    p.add_argument("--m", type=int, default=None, help="token count (default: the workload's first M)")
    p.add_argument("--repeats", type=int, default=5, help="extra timed regions of K steps (median reported)")
    p.add_argument("--e2e-steps", type=int, default=50)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sub", action="store_true", help="skip the sub-records")
    p.add_argument("--reference-budget-s", type=float, default=150.0,
                   help="CPU seconds the reference (oracle) arm may spend in total")
    p.add_argument("--profile-kernel", choices=["gemv", "gemm", "quantize", "act_scale"], default=None,
                   help="only run --launches launches of one kernel on layer --layer of the workload (for ncu)")
    p.add_argument("--layer", type=int, default=0)
    p.add_argument("--launches", type=int, default=4)
    return p.parse_args(argv)


# ----------------------------------------------------------------------------- algorithmic work per launch
def packed_bytes(N, K):
    """Bytes of packed layout v2: per (16-row tile, group pair) 2048 codes + 64 scales + 16 zeros."""
    return (-(-N // 16)) * (-(-(K // GROUP) // 2)) * (2048 + 64 + 16)


def bytes_act_scale(M, K):          # read x twice, write x' and s
    return 3 * 2 * M * K + 4 * K


def bytes_quantize(N, K):           # read fp16 W and s, write packed
    return 2 * N * K + 4 * K + packed_bytes(N, K)


def bytes_linear(M, N, K):          # read packed W and x', write y
    return packed_bytes(N, K) + 2 * M * K + 2 * M * N


def flops_linear(M, N, K):
    return 2 * M * N * K


def rotation_sets(bytes_per_set, l2_bytes):
    """Copies of a working set needed so that the copies together are at least 4x the L2 size."""
    return max(2, int(math.ceil(4.0 * l2_bytes / max(bytes_per_set, 1))))


def exact_step_plan(steps, R):
    """(full replays of an R-step graph, remainder steps): R * full + rem == steps exactly."""
    R = max(1, min(R, steps)) if steps > 0 else 1
    return R, steps // R, steps % R


# ----------------------------------------------------------------------------- clocks sampler
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)

    def summary(self, t0, t1):
        rows = [l for (t, l) in self.lines if t0 <= t <= t1] or [l for (_, l) in self.lines]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in rows:
            parts = [x.strip() for x in l.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_init(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group("nccl" if args.impl == "ours" else "gloo",
                                timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(value: float, world: int, device: str = "cuda") -> float:
    """Max over ranks (timing is taken as the slowest rank's device time)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(weights_per_step: int, steps: int, ms_max: float, world: int) -> float:
    """Whole-job fp16-equivalent weight GB/s: every rank processes its own replica."""
    return world * 2.0 * weights_per_step * steps / (ms_max * 1e-3) / 1e9


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- host description
def host_cpu():
    """CPU model, core count and the BLAS thread pools NumPy will use."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    blas = []
    try:
        from threadpoolctl import threadpool_info
        blas = [{"api": d.get("internal_api"), "threads": d.get("num_threads")} for d in threadpool_info()]
    except Exception:
        pass
    return {"cpu_model": model, "cpu_count": os.cpu_count(), "blas": blas}


# ----------------------------------------------------------------------------- the oracle on the host
def oracle_decode_inputs(wl, M):
    """Seeded inputs of every layer and the oracle's quantized weights (outside any timed region)."""
    from oracle import awq_oracle as O
    out = []
    for i in range(len(wl.layers)):
        x, W = workloads.layer_inputs(wl, i, M)
        s = O.activation_scale(x)
        xs = O.scale_activations(x, s)
        q, S, z = O.quantize_groups(O.fold_weights(W, s))
        out.append((xs, q, S, z))
    return out


def oracle_decode_step(layers, rows):
    """The oracle's W4A16 linear layer (dequantize + float64 matmul) on the first `rows` rows of
    every layer; returns the number of weights processed."""
    from oracle import awq_oracle as O
    n = 0
    for (xs, q, S, z) in layers:
        r = min(rows, q.shape[0])
        O.linear(xs, O.dequantize(q[:r], S[:r], z[:r]))
        n += r * q.shape[1]
    return n


def cpu_baseline(layers, target_s=15.0):
    """The oracle as it stands, on every host core (BLAS threads = os.cpu_count()), on a bounded row
    sample of the workload; value in the headline metric's unit."""
    from threadpoolctl import threadpool_limits
    cores = os.cpu_count() or 1
    max_rows = max(q.shape[0] for (_, q, _, _) in layers)
    with threadpool_limits(limits=cores):
        t = time.perf_counter()
        oracle_decode_step(layers, 128)
        probe = time.perf_counter() - t
        rows = int(max(128, min(max_rows, 128 * (target_s / 3) / max(probe, 1e-3))))
        t = time.perf_counter()
        w, reps = 0, 0
        while True:
            w += oracle_decode_step(layers, rows)
            reps += 1
            if time.perf_counter() - t >= 0.8 * target_s or reps >= 50:
                break
        dt = time.perf_counter() - t
    hc = host_cpu()
    return {"value": 2.0 * w / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"oracle W4A16 linear (NumPy dequantize + float64 matmul, BLAS on {cores} threads) on the "
                      f"first {rows} rows of every layer, {reps} pass(es): {w} weights in {dt:.2f} s; "
                      f"value = fp16-equivalent weight bytes (2/weight) per second; weights quantized beforehand",
            "host": hc}


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, world, rank):
    if rank != 0:
        dist_done(world)
        return
    from threadpoolctl import threadpool_limits
    wl = workloads.WORKLOADS[args.workload]
    M = args.m or wl.Ms[0]
    layers = oracle_decode_inputs(wl, M)
    cores = os.cpu_count() or 1
    total_steps = args.steps + args.warmup
    with threadpool_limits(limits=cores):
        t = time.perf_counter()
        oracle_decode_step(layers, 64)
        probe = time.perf_counter() - t
        max_rows = max(q.shape[0] for (_, q, _, _) in layers)
        rows = int(max(16, min(max_rows, 64 * (args.reference_budget_s / max(total_steps, 1)) / max(probe, 1e-4))))
        for _ in range(args.warmup):
            oracle_decode_step(layers, rows)
        t = time.perf_counter()
        w = 0
        for _ in range(args.steps):
            w += oracle_decode_step(layers, rows)
        dt = time.perf_counter() - t
    value = 2.0 * w / dt / 1e9
    line = {
        "impl": "reference", "metric": metric_name(M), "value": value, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": bench_config(wl, M),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"oracle W4A16 linear on the first {rows} rows of each layer per step",
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    dist_done(world)


def metric_name(M):
    return "W4A16 g128 effective weight GB/s (decode GEMV) and TFLOP/s (prefill GEMM), % roofline"


def bench_config(wl, M, n_sets=None, set_mb=None):
    decode = M <= 32
    lin = "decode GEMV (awq_w4a16_gemv)" if decode else "prefill GEMM (awq_w4a16_gemm)"
    cfg = {"workload": wl.name, "M": M,
           "layers": [{"name": l.name, "K": l.K, "N": l.N} for l in wl.layers],
           "step": f"one {lin} launch per layer on weights folded and quantized once before timing",
           "weights": "int4, group 128 along K, fp16 scale, 4-bit zero point (packed layout v2)",
           "accumulate": "f32",
           "value": ("fp16-equivalent weight bytes (2 per weight) per second" if decode
                     else "dense FLOP/s (2*M*N*K per layer)")}
    if n_sets is not None:
        cfg["l2"] = (f"inputs larger than L2: packed weights rotated over {n_sets} copies of {set_mb:.1f} MB "
                     f"({n_sets * set_mb:.0f} MB >= 4x the L2 size) between steps")
    return cfg


# ----------------------------------------------------------------------------- profile records
def code_hash(src):
    """SHA-256 (first 16 hex digits) of C++/CUDA source text with comments and whitespace removed,
    so that only a change of the code itself counts."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    src = re.sub(r"\s+", "", src)
    return hashlib.sha256(src.encode()).hexdigest()[:16]


def kernel_source_hash(name):
    """code_hash of a kernel source file of the package (None if it is missing)."""
    p = os.path.join(ROOT, "weight_only_quantization_w4a16_b200", "csrc", name)
    try:
        return code_hash(open(p).read())
    except OSError:
        return None


def profile_traffic(kernel_file, workload, M):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this workload and M
    and the kernel source is unchanged since."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        d = json.load(open(p))
    except (OSError, ValueError):
        return None
    if d.get("_workload") != workload or d.get("_M") != M:
        return None
    e = d.get(kernel_file)
    if not e or e.get("source_sha256_16") != kernel_source_hash(kernel_file):
        return None
    return e


# ----------------------------------------------------------------------------- ours
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d.get("hbm_gbs", 6650.0)), float(d.get("bf16_tflops", 1590.0)),
                float(d.get("bf16_tflops_sustained", 1400.0)), "of measured")
    return 6650.0, 1590.0, 1400.0, "of fallback"


class GraphTimer:
    """Captures launches into CUDA graphs on one stream and times replays with CUDA events."""

    def __init__(self, torch, stream):
        self.torch, self.stream = torch, stream

    def capture(self, fn, count):
        g = self.torch.cuda.CUDAGraph()
        with self.torch.cuda.graph(g, stream=self.stream):
            for i in range(count):
                fn(i)
        return g

    def time(self, graphs, repeats=1):
        """ms of one pass over `graphs` (a list of (graph, replays)), for each of `repeats` passes."""
        torch = self.torch
        out = []
        for _ in range(repeats):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            for g, n in graphs:
                for _ in range(n):
                    g.replay()
            e1.record(self.stream)
            e1.synchronize()
            out.append(e0.elapsed_time(e1))
        return out


def per_launch_us(timer, fn, launches=64, repeats=5):
    """Median µs per launch of `fn(i)` over `launches` back-to-back launches in one graph."""
    with timer.torch.cuda.stream(timer.stream):
        for i in range(3):
            fn(i)
        timer.stream.synchronize()
        g = timer.capture(fn, launches)
        timer.time([(g, 1)])
        ms = timer.time([(g, 1)], repeats)
    return 1e3 * statistics.median(ms) / launches, g


def run_ours(args, world, rank, local):
    import torch
    import weight_only_quantization_w4a16_b200 as P

    P.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 0) or L2_BYTES_DEFAULT)
    wl = workloads.WORKLOADS[args.workload]
    M = args.m or wl.Ms[0]
    decode = M <= 32
    hbm_peak, tc_peak, tc_sus, peak_src = load_peaks()
    stream = torch.cuda.Stream(device=dev)
    timer = GraphTimer(torch, stream)
    lin = P.awq_w4a16_gemv if decode else P.awq_w4a16_gemm

    # ---------------------------------------------------------------- set-up (not timed)
    host = [workloads.layer_inputs(wl, i, M) for i in range(len(wl.layers))]
    L = []
    with torch.cuda.stream(stream):
        for (x, W), layer in zip(host, wl.layers):
            N, K = layer.N, layer.K
            d = {"N": N, "K": K, "x": torch.from_numpy(x).to(dev)}
            Wd = torch.from_numpy(W).to(dev)
            d["s"], d["xs"] = P.awq_activation_scale(d["x"], 0.5)
            d["packed"] = [P.awq_quantize_g128(Wd, d["s"])]
            d["y"] = torch.empty((M, N), dtype=torch.float16, device=dev)
            del Wd
            L.append(d)
        set_bytes = sum(packed_bytes(d["N"], d["K"]) for d in L)
        n_sets = rotation_sets(set_bytes, l2)
        for d in L:
            d["packed"] += [tuple(t.clone() for t in d["packed"][0]) for _ in range(n_sets - 1)]
        stream.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK

    def step(i):
        """One decode (or prefill) pass over every layer, on packed copy set i mod n_sets."""
        for d in L:
            lin(d["xs"], *d["packed"][i % n_sets], d["N"], d["y"])

    # ---------------------------------------------------------------- warm-up and the timed region
    K_steps, W_steps = args.steps, max(3, args.warmup)
    R, full, rem = exact_step_plan(K_steps, 50)
    with torch.cuda.stream(stream):
        for i in range(2):
            step(i)                       # sets kernel attributes before any capture
        stream.synchronize()
        g_main = timer.capture(step, R)
        g_rem = timer.capture(step, rem) if rem else None
        g_warm = timer.capture(step, W_steps)
    plan = [(g_main, full)] + ([(g_rem, 1)] if g_rem is not None else [])
    gpu_uuid = None
    try:
        gpu_uuid = str(props.uuid)
        gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else "GPU-" + gpu_uuid
    except Exception:
        gpu_uuid = str(local)
    clocks = ClockSampler(gpu_uuid)
    with torch.cuda.stream(stream):
        timer.time([(g_warm, 1)])        # W warm-up steps
        stream.synchronize()
        dist_barrier(world)
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.25)
        t_wall0 = time.time()
        ms_total = timer.time(plan)[0]   # exactly K steps
        torch.cuda.synchronize()
        dist_barrier(world)
        # repeats of the same K-step region, and a sustained run long enough for the clock samples
        rep_ms = timer.time(plan, max(1, args.repeats))
        sus_steps = 0
        sus_ms = 0.0
        t_s = time.time()
        while time.time() - t_s < 1.5:
            sus_ms += timer.time([(g_main, 20)])[0]
            sus_steps += 20 * R
        t_wall1 = time.time()
        clocks.stop()
    assert P.awq_poll_device_status() == P.AWQ_OK, "a kernel reported a timeout"

    ms_total = dist_max(ms_total, world)
    ms_step = ms_total / K_steps
    weights_per_step = sum(d["N"] * d["K"] for d in L)
    alg_bytes_step = sum(bytes_linear(M, d["N"], d["K"]) for d in L)
    flops_step = sum(flops_linear(M, d["N"], d["K"]) for d in L)
    if decode:
        value = weak_scaling_value(weights_per_step, K_steps, ms_total, world)
        unit = "GB/s"
    else:
        value = world * flops_step * K_steps / (ms_total * 1e-3) / 1e12
        unit = "TFLOP/s"
    kfile = "awq_gemv.cuh" if decode else "awq_gemm.cuh"
    tr = profile_traffic(kfile, wl.name, M)
    if decode:
        achieved = alg_bytes_step / (ms_step * 1e-3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak,
                "traffic": tr["bytes_per_step"] if tr else None, "kernel": "awq_gemv_kernel",
                "peak_source": peak_src + " (HBM copy)",
                "algorithmic_bytes": "per step: sum over layers of packed(N,K) + 2*M*K + 2*M*N, "
                                     "packed(N,K) = ceil(N/16)*ceil(K/256)*2128; %d bytes" % alg_bytes_step,
                "note": "the step is the decode kernel's launches only: achieved = algorithmic bytes of a "
                        "step / the step's device time"}
    else:
        achieved = flops_step / (ms_step * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tc_sus, "unit": "TFLOP/s", "frac": achieved / tc_sus,
                "traffic": tr["bytes_per_step"] if tr else None, "kernel": "awq_gemm_kernel",
                "peak_source": peak_src + " (bf16 sustained; fp16 dense has the same nominal rate)",
                "frac_of_burst": achieved / tc_peak}

    # ---------------------------------------------------------------- sub-records
    sub = None
    if not args.no_sub and rank == 0 and world == 1:
        sub = sub_records(torch, P, timer, dev, l2, hbm_peak, tc_peak, tc_sus, peak_src, wl, M, L, n_sets)

    # ---------------------------------------------------------------- end to end (host buffers, public API)
    e2e = None
    if not args.no_e2e:
        e2e = end_to_end(torch, P, stream, host, L, M, args.e2e_steps, world, decode)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(oracle_decode_inputs(wl, M)) if decode else None

    config = bench_config(wl, M, n_sets, set_bytes / 1e6)
    if not decode:   # the token tile and K split the prefill kernel took for each layer
        config["plan"] = [{"layer": l.name, "token_tile": bt, "k_split": ks, "split_tiles": nsplit}
                          for l in wl.layers for bt, ks, nsplit in [P.awq_gemm_plan(M, l.N, l.K)]]
    line = {
        "metric": metric_name(M), "value": value, "unit": unit, "n_gpus": world, "steps": K_steps,
        "warmup": W_steps, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": config, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": K_steps * len(L),
        "clocks": clocks.summary(t_wall0, t_wall1),
        "repeats": {"ms_per_step": [m / K_steps for m in rep_ms], "median_ms_per_step": statistics.median(rep_ms) / K_steps,
                    "median_value": (weak_scaling_value(weights_per_step, K_steps, statistics.median(rep_ms), world)
                                     if decode else world * flops_step * K_steps / statistics.median(rep_ms) / 1e9)},
        "sustained": {"steps": sus_steps, "ms_per_step": sus_ms / max(sus_steps, 1),
                      "value": (weak_scaling_value(weights_per_step, sus_steps, sus_ms, world) if decode
                                else world * flops_step * sus_steps / sus_ms / 1e9),
                      "note": "about 1.5 s of back-to-back steps, during which the clocks are sampled"},
        "timing": ("CUDA events on the launching stream around exactly K steps (graph replays of %d-step "
                   "graphs%s), after W warm-up steps; packed weights rotated between steps" %
                   (R, " plus one %d-step graph" % rem if rem else "")),
        "sub": sub,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    dist_done(world)


def sub_records(torch, P, timer, dev, l2, hbm_peak, tc_peak, tc_sus, peak_src, wl, M, L, n_sets):
    """Per-kernel records, each timed alone (back-to-back launches in a graph, median of 5)."""
    out = {}
    rec_layers = []
    # decode GEMV per layer of this workload (its own rotation already in L)
    if M <= 32:
        for d in L:
            us, g = per_launch_us(timer, lambda i, d=d: P.awq_w4a16_gemv(d["xs"], *d["packed"][i % n_sets], d["N"],
                                                                         d["y"]))
            del g
            b = bytes_linear(M, d["N"], d["K"])
            rec_layers.append({"layer": f"{wl.name}/{d['N']}x{d['K']}", "M": M, "us": us,
                               "GBps": b / us / 1e3, "frac": b / us / 1e3 / hbm_peak,
                               "effective_weight_GBps": 2 * d["N"] * d["K"] / us / 1e3})
    # the two Llama-2-70B layers: decode GEMV at M = 1 and the quantizer over the full fp16 layer
    wl70 = workloads.WORKLOADS["llama2_70b_layers"]
    qrec = []
    for li, layer in enumerate(wl70.layers):
        x, W = workloads.layer_inputs(wl70, li, 1)
        N, K = layer.N, layer.K
        with torch.cuda.stream(timer.stream):
            xd = torch.from_numpy(x).to(dev)
            Wd = torch.from_numpy(W).to(dev)
            s, xs = P.awq_activation_scale(xd, 0.5)
            packed = P.alloc_packed(N, K, dev)
            us_q, g = per_launch_us(timer, lambda i: P.awq_quantize_g128(Wd, s, packed), launches=10)
            del g
            bq = bytes_quantize(N, K)
            qrec.append({"layer": f"llama2_70b/{N}x{K}", "us": us_q, "GBps": bq / us_q / 1e3,
                         "frac": bq / us_q / 1e3 / hbm_peak, "algorithmic_bytes": bq})
            nset = rotation_sets(packed_bytes(N, K), l2)
            copies = [packed] + [tuple(t.clone() for t in packed) for _ in range(nset - 1)]
            del Wd
            y = torch.empty((1, N), dtype=torch.float16, device=dev)
            us, g = per_launch_us(timer, lambda i: P.awq_w4a16_gemv(xs, *copies[i % nset], N, y))
            del g, copies
        b = bytes_linear(1, N, K)
        rec_layers.append({"layer": f"llama2_70b/{N}x{K}", "M": 1, "us": us, "GBps": b / us / 1e3,
                           "frac": b / us / 1e3 / hbm_peak, "effective_weight_GBps": 2 * N * K / us / 1e3})
    out["gemv_layers"] = {"kernel": "awq_gemv_kernel", "bound": "hbm", "peak": hbm_peak,
                          "peak_source": peak_src + " (HBM copy)", "records": rec_layers,
                          "note": "each layer alone: 64 launches back to back in a CUDA graph over packed copies "
                                  "rotated through >= 4x L2; algorithmic bytes packed(N,K) + 2MK + 2MN"}
    out["quantize"] = {"kernel": "awq_quantize_g128_kernel", "bound": "hbm", "peak": hbm_peak,
                       "peak_source": peak_src + " (HBM copy)", "records": qrec,
                       "note": "fold + quantize of the full fp16 layer (10 launches back to back); algorithmic "
                               "bytes 2NK + 4K + packed(N,K)"}
    # prefill GEMM: Llama-3-8B gate+up at M = 4096
    wl8 = workloads.WORKLOADS["llama3_8b_prefill"]
    li = 2
    Mg = 4096
    x, W = workloads.layer_inputs(wl8, li, Mg)
    N, K = wl8.layers[li].N, wl8.layers[li].K
    with torch.cuda.stream(timer.stream):
        s, xs = P.awq_activation_scale(torch.from_numpy(x).to(dev), 0.5)
        Wd = torch.from_numpy(W).to(dev)
        packed = P.awq_quantize_g128(Wd, s)
        del Wd
        y = torch.empty((Mg, N), dtype=torch.float16, device=dev)
        us, g = per_launch_us(timer, lambda i: P.awq_w4a16_gemm(xs, *packed, N, y), launches=20)
        del g
    tf = flops_linear(Mg, N, K) / us / 1e6
    out["gemm"] = {"kernel": "awq_gemm_kernel", "bound": "tensor", "layer": f"llama3_8b/{N}x{K}", "M": Mg,
                   "us": us, "TFLOPs": tf, "peak": tc_sus, "frac": tf / tc_sus, "frac_of_burst": tf / tc_peak,
                   "peak_source": peak_src + " (bf16 sustained for 20 back-to-back launches; burst also given)"}
    # activation statistic + scaling: 4096 tokens x 4096 channels, rotated over 5 activation copies
    xa = [torch.from_numpy(workloads.make_activations(0, 4, 0, 4096, 4096)).to(dev) for _ in range(5)]
    sa = torch.empty(4096, dtype=torch.float32, device=dev)
    xsa = torch.empty((4096, 4096), dtype=torch.float16, device=dev)
    us, g = per_launch_us(timer, lambda i: P.awq_activation_scale(xa[i % 5], 0.5, sa, xsa), launches=20)
    del g
    ba = bytes_act_scale(4096, 4096)
    out["act_scale"] = {"kernel": "awq_act_scale_kernel", "bound": "hbm", "shape": "M=4096, K=4096", "us": us,
                        "GBps": ba / us / 1e3, "frac": ba / us / 1e3 / hbm_peak, "peak": hbm_peak}
    # decode kernel vs prefill kernel on the batched-decode shapes, and what awq_w4a16_linear picks
    if M == 1 and wl.name == "llama2_7b_decode_m1":
        out["crossover"] = crossover(torch, P, timer, dev, l2)
    # a dependent decode chain of one Llama-2-7B block at M = 1: scale -> fused q/k/v (split) ->
    # scale -> o_proj -> scale -> fused gate+up (SiLU * up) -> scale -> down, each layer fed by the
    # previous output (q stands in for the attention output), weights rotated through >= 4x L2
    if M == 1 and wl.name == "llama2_7b_decode_m1":
        out["decode_layer_chain"] = decode_layer_chain(torch, P, timer, dev, l2, hbm_peak, wl)
    # one pass of every row of the path on this workload: a1 + a2 + linear per layer (full fp16 W read)
    if M <= 32:
        Ws = [torch.from_numpy(workloads.layer_inputs(wl, i, M)[1]).to(dev) for i in range(len(L))]
        scratch = [P.alloc_packed(d["N"], d["K"], dev) for d in L]

        def full_step(i):
            for d, Wd, pk in zip(L, Ws, scratch):
                P.awq_activation_scale(d["x"], 0.5, d["s"], d["xs"])
                P.awq_quantize_g128(Wd, d["s"], pk)
                P.awq_w4a16_gemv(d["xs"], *pk, d["N"], d["y"])
        us, g = per_launch_us(timer, full_step, launches=8)
        del g
        out["full_path"] = {"us_per_step": us, "launches_per_step": 3 * len(L),
                            "note": "activation statistic + fold/quantize + decode GEMV for every layer of the "
                                    "workload (fp16 weights re-quantized every step)"}
    return out


def crossover(torch, P, timer, dev, l2, Ms=(4, 8, 16, 32)):
    """µs per launch of the decode kernel, the prefill kernel and the dispatching call per layer and M."""
    wl3 = workloads.WORKLOADS["llama2_7b_decode_batched"]
    recs = []
    for li, layer in enumerate(wl3.layers):
        x, W = workloads.layer_inputs(wl3, li, max(Ms))
        N, K = layer.N, layer.K
        with torch.cuda.stream(timer.stream):
            s, xs = P.awq_activation_scale(torch.from_numpy(x).to(dev), 0.5)
            Wd = torch.from_numpy(W).to(dev)
            packed = P.awq_quantize_g128(Wd, s)
            del Wd
            nset = rotation_sets(packed_bytes(N, K), l2)
            copies = [packed] + [tuple(t.clone() for t in packed) for _ in range(nset - 1)]
            for Mx in Ms:
                xm = xs[:Mx].contiguous()
                y = torch.empty((Mx, N), dtype=torch.float16, device=dev)
                r = {"layer": f"{wl3.name}/{N}x{K}", "M": Mx}
                for name, fn in (("gemv", P.awq_w4a16_gemv), ("gemm", P.awq_w4a16_gemm), ("linear", P.awq_w4a16_linear)):
                    us, g = per_launch_us(timer, lambda i, fn=fn: fn(xm, *copies[i % nset], N, y), launches=16)
                    del g
                    r[name + "_us"] = us
                r["faster"] = "gemv" if r["gemv_us"] <= r["gemm_us"] else "gemm"
                recs.append(r)
            del copies
    return {"records": recs,
            "note": "16 launches back to back in a CUDA graph over packed copies rotated through >= 4x L2, median "
                    "of 5; awq_w4a16_linear takes the decode kernel for M <= 32 unless its full-size configuration "
                    "does not fit in shared memory"}


def decode_layer_chain(torch, P, timer, dev, l2, hbm_peak, wl):
    """Times the dependent chain of a Llama-2-7B block's linear layers at M = 1 (see sub_records)."""
    layers = []
    for li, layer in enumerate(wl.layers):
        x, W = workloads.layer_inputs(wl, li, 1)
        with torch.cuda.stream(timer.stream):
            s, _ = P.awq_activation_scale(torch.from_numpy(x).to(dev), 0.5, want_scaled=False)
            Wd = torch.from_numpy(W).to(dev)
            pk = P.awq_quantize_g128(Wd, s)
            del Wd
        layers.append({"N": layer.N, "K": layer.K, "s": s, "packed": [pk]})
    nset = rotation_sets(sum(packed_bytes(d["N"], d["K"]) for d in layers), l2)
    for d in layers:
        d["packed"] += [tuple(t.clone() for t in d["packed"][0]) for _ in range(nset - 1)]
    qkv, o, gu, down = layers
    x0 = torch.from_numpy(workloads.layer_inputs(wl, 0, 1)[0]).to(dev)
    xs = torch.empty((1, 11008), dtype=torch.float16, device=dev)
    q, k, v = (torch.empty((1, 4096), dtype=torch.float16, device=dev) for _ in range(3))
    yo = torch.empty((1, 4096), dtype=torch.float16, device=dev)
    h = torch.empty((1, 11008), dtype=torch.float16, device=dev)
    y = torch.empty((1, 4096), dtype=torch.float16, device=dev)

    def chain(i):
        c = i % nset
        P.awq_scale_activations(x0, qkv["s"], xs[:, :4096])
        P.awq_w4a16_linear_qkv(xs[:, :4096], *qkv["packed"][c], 4096, 4096, out=(q, k, v))
        P.awq_scale_activations(q, o["s"], xs[:, :4096])
        P.awq_w4a16_gemv(xs[:, :4096], *o["packed"][c], 4096, yo)
        P.awq_scale_activations(yo, gu["s"], xs[:, :4096])
        P.awq_w4a16_linear_silu_mul(xs[:, :4096], *gu["packed"][c], 11008, h)
        P.awq_scale_activations(h, down["s"], xs)
        P.awq_w4a16_gemv(xs, *down["packed"][c], 4096, y)

    us, g = per_launch_us(timer, chain, launches=32)
    del g
    wbytes = sum(2 * d["N"] * d["K"] for d in layers)
    alg = sum(bytes_linear(1, d["N"], d["K"]) for d in layers)
    return {"us_per_step": us, "launches_per_step": 8, "effective_weight_GBps": wbytes / us / 1e3,
            "GBps": alg / us / 1e3, "frac": alg / us / 1e3 / hbm_peak,
            "note": "one Llama-2-7B block's linear layers at M = 1 as a dependent chain in a CUDA graph with "
                    "programmatic dependent launch: scale + fused q/k/v, scale + o_proj, scale + fused "
                    "gate/up SiLU*up, scale + down; 32 steps back to back over rotated weights"}


def end_to_end(torch, P, stream, host, L, M, steps, world, decode):
    """The same metric through the Python binding with host buffers: every step copies each layer's
    activations in from pinned host memory, scales them by the stored s and runs the linear layer
    (AWQLinear), and copies y out. The packed weights stay resident, as a deployed model's do."""
    pin_x = [torch.from_numpy(x).pin_memory() for (x, _) in host]
    y_host = [torch.empty((M, d["N"]), dtype=torch.float16).pin_memory() for d in L]
    layers = [P.AWQLinear(*d["packed"][0], d["s"], d["N"], d["K"]) for d in L]
    h2d = sum(x.numel() * 2 for x in pin_x)
    d2h = sum(y.numel() * 2 for y in y_host)

    def e2e_step():
        for xh, d, lay, yh in zip(pin_x, L, layers, y_host):
            d["x"].copy_(xh, non_blocking=True)
            lay(d["x"], d["y"])
            yh.copy_(d["y"], non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            e2e_step()
        stream.synchronize()
        dist_barrier(world)
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(steps):
            e2e_step()
        a1.record(stream)
        a1.synchronize()
    ms = dist_max(a0.elapsed_time(a1), world)
    weights = sum(d["N"] * d["K"] for d in L)
    flops = sum(flops_linear(M, d["N"], d["K"]) for d in L)
    v = weak_scaling_value(weights, steps, ms, world) if decode else world * flops * steps / (ms * 1e-3) / 1e12
    return {"value": v, "unit": "GB/s" if decode else "TFLOP/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps,
            "note": "eager calls through the Python binding (AWQLinear: scale x by the stored s, then the linear "
                    "kernel) with pinned-host x copied in and y copied out every step; packed weights resident"}


def profile_kernel(args):
    """A few launches of one kernel on one layer of a workload, inputs prepared beforehand: the small,
    self-contained case an ncu capture of that kernel runs on."""
    import torch
    import weight_only_quantization_w4a16_b200 as P
    P.load_library()
    torch.cuda.set_device(0)
    wl = workloads.WORKLOADS[args.workload]
    M = args.m if args.m is not None else wl.Ms[0]
    layer = wl.layers[args.layer]
    x, W = workloads.layer_inputs(wl, args.layer, M)
    xd, Wd = torch.from_numpy(x).cuda(), torch.from_numpy(W).cuda()
    s, xs = P.awq_activation_scale(xd, 0.5)
    packed = P.awq_quantize_g128(Wd, s)
    y = torch.empty((M, layer.N), dtype=torch.float16, device="cuda")
    for _ in range(args.launches):
        if args.profile_kernel == "gemv":
            P.awq_w4a16_gemv(xs, *packed, layer.N, y)
        elif args.profile_kernel == "gemm":
            P.awq_w4a16_gemm(xs, *packed, layer.N, y)
        elif args.profile_kernel == "quantize":
            P.awq_quantize_g128(Wd, s, packed)
        else:
            P.awq_activation_scale(xd, 0.5, s, xs)
    torch.cuda.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK
    print(f"{args.profile_kernel}: {args.launches} launches on {wl.name} layer {args.layer} "
          f"({layer.N}x{layer.K}), M = {M}", flush=True)


def main():
    args = parse_args()
    if args.profile_kernel:
        profile_kernel(args)
        return
    world, rank, local = dist_init(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
