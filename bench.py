#!/usr/bin/env python
"""Benchmark of the AWQ W4A16 g128 hot path on B200.

One step = one pass of the whole path over one batch of synthetic input: for
every layer of the workload, the activation statistic and scaling (a1), the
fold + group quantizer (a2) and the W4A16 linear layer (a3 decode for
M <= 32, a4 prefill otherwise). The default workload is the Llama-2-7B decode
GEMV set at M = 1 (four layers: 4096x12288, 4096x4096, 4096x22016,
11008x4096). Its fp16 weights (405 MB per step) exceed the 126 MB L2, so
every step streams from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs its own replica (weak scaling, no data-path
collective); timing is on the device with CUDA events, max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
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


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=8000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="llama2_7b_decode_m1", choices=workloads.workload_names())
    p.add_argument("--m", type=int, default=None, help="token count (default: the workload's first M)")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--graph-steps", type=int, default=8, help="steps per captured CUDA graph")
    p.add_argument("--reference-budget-s", type=float, default=150.0,
                   help="CPU seconds the reference (oracle) arm may spend in total")
    return p.parse_args()


# ----------------------------------------------------------------------------- algorithmic work per launch
def packed_bytes(N, K):
    Np = -(-N // 128) * 128
    return Np * K // 2 + Np * (K // GROUP) * 2 + Np * (K // GROUP) // 2


def bytes_act_scale(M, K):          # read x twice, write x' and s
    return 3 * 2 * M * K + 4 * K


def bytes_quantize(N, K):           # read fp16 W and s, write packed
    return 2 * N * K + 4 * K + packed_bytes(N, K)


def bytes_linear(M, N, K):          # read packed W and x', write y
    return packed_bytes(N, K) + 2 * M * K + 2 * M * N


def flops_linear(M, N, K):
    return 2 * M * N * K


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


# ----------------------------------------------------------------------------- CPU oracle baseline
def oracle_sample_step(layers_data, rows_per_layer):
    """The oracle on a bounded sample: every layer's activation statistic (full
    x), fold + quantize + dequantize + matmul of the first `rows` rows."""
    from oracle import awq_oracle as O
    weights = 0
    for (x, W) in layers_data:
        rows = min(rows_per_layer, W.shape[0])
        s = O.activation_scale(x)
        xs = O.scale_activations(x, s)
        q, S, z = O.quantize_groups(O.fold_weights(W[:rows], s))
        O.linear(xs, O.dequantize(q, S, z))
        weights += rows * W.shape[1]
    return weights


def cpu_baseline(layers_data, target_s=12.0, threads=1):
    """The oracle, single-threaded, on about `target_s` seconds of the workload: the first rows of
    every layer (all rows when that is not enough), repeated until the target is reached."""
    from threadpoolctl import threadpool_limits
    max_rows = max(W.shape[0] for _, W in layers_data)
    with threadpool_limits(limits=threads):
        t = time.perf_counter()
        oracle_sample_step(layers_data, 128)
        probe = time.perf_counter() - t
        rows = int(max(128, min(max_rows, 128 * target_s / max(probe, 1e-3))))
        t = time.perf_counter()
        w, reps = 0, 0
        while True:
            w += oracle_sample_step(layers_data, rows)
            reps += 1
            if time.perf_counter() - t >= 0.8 * target_s or reps >= 20:
                break
        dt = time.perf_counter() - t
    return {"value": 2.0 * w / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"oracle (NumPy, {threads} thread) on the first {rows} rows of every layer, {reps} pass(es) "
                      f"(fold + quantize + dequantize + float64 matmul; activation statistic over all of x); "
                      f"{w} weights in {dt:.2f} s; value = fp16-equivalent weight bytes (2/weight) per second"}


# ----------------------------------------------------------------------------- reference arm (the oracle)
def run_reference(args, world, rank):
    if rank != 0:
        dist_done(world)
        return
    wl = workloads.WORKLOADS[args.workload]
    M = args.m or wl.Ms[0]
    data = [workloads.layer_inputs(wl, i, M) for i in range(len(wl.layers))]
    from threadpoolctl import threadpool_limits
    total_steps = args.steps + args.warmup
    budget_s = args.reference_budget_s
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        oracle_sample_step(data, 64)
        probe = time.perf_counter() - t
        rows = int(max(16, min(4096, 64 * (budget_s / total_steps) / max(probe, 1e-4))))
        for _ in range(args.warmup):
            oracle_sample_step(data, rows)
        t = time.perf_counter()
        w = 0
        for _ in range(args.steps):
            w += oracle_sample_step(data, rows)
        dt = time.perf_counter() - t
    value = 2.0 * w / dt / 1e9
    line = {
        "impl": "reference", "metric": metric_name(M), "value": value, "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64",
        "data": "synthetic", "config": bench_config(wl, M),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"oracle on the first {rows} rows of each layer per step"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    dist_done(world)


def metric_name(M):
    return "W4A16 g128 effective weight GB/s (decode GEMV) and TFLOP/s (prefill GEMM), % roofline"


def bench_config(wl, M):
    lin = "decode GEMV (a3)" if M <= 32 else "prefill GEMM (a4)"
    return {"workload": wl.name, "M": M,
            "layers": [{"name": l.name, "K": l.K, "N": l.N} for l in wl.layers],
            "step": "per layer: activation statistic + scaling (a1), fold + 4-bit g128 quantizer (a2), " + lin,
            "weights": "int4, group 128 along K, fp16 scale, 4-bit zero point",
            "accumulate": "f32",
            "l2": "inputs larger than L2 (fp16 weights of the step: %.0f MB vs 126 MB L2)"
                  % (sum(2 * l.N * l.K for l in wl.layers) / 1e6),
            "value": "fp16-equivalent weight bytes (2 per weight) per second over the whole step"}


# ----------------------------------------------------------------------------- ours
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


def run_ours(args, world, rank, local):
    import torch
    import weight_only_quantization_w4a16_b200 as P

    P.load_library()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = workloads.WORKLOADS[args.workload]
    M = args.m or wl.Ms[0]
    decode = M <= 32

    host = [workloads.layer_inputs(wl, i, M) for i in range(len(wl.layers))]
    L = []
    for (x, W), layer in zip(host, wl.layers):
        N, K = layer.N, layer.K
        d = {"N": N, "K": K,
             "x": torch.from_numpy(x).to(dev), "W": torch.from_numpy(W).to(dev),
             "s": torch.empty(K, dtype=torch.float32, device=dev),
             "xs": torch.empty((M, K), dtype=torch.float16, device=dev),
             "y": torch.empty((M, N), dtype=torch.float16, device=dev)}
        d["packed"] = P.alloc_packed(N, K, dev)
        L.append(d)

    lin = P.awq_w4a16_gemv if decode else P.awq_w4a16_gemm

    kernels = ["act_scale", "quantize", "gemv" if decode else "gemm"]

    def step(events=None):
        """One pass of the path over all layers, grouped by kernel: a1 for every layer, then a2,
        then the linear layer (the layers are independent). `events` (4 per step) mark the groups."""
        if events is not None:
            events[0].record()
        for d in L:
            P.awq_activation_scale(d["x"], 0.5, d["s"], d["xs"])
        if events is not None:
            events[1].record()
        for d in L:
            P.awq_quantize_g128(d["W"], d["s"], d["packed"])
        if events is not None:
            events[2].record()
        for d in L:
            lin(d["xs"], *d["packed"], d["N"], d["y"])
        if events is not None:
            events[3].record()

    stream = torch.cuda.Stream(device=dev)
    R = max(1, args.graph_steps)
    with torch.cuda.stream(stream):
        for _ in range(3):          # eager warm-up: sets kernel attributes before capture
            step()
        stream.synchronize()
        assert P.awq_poll_device_status() == P.AWQ_OK
        g_plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_plain, stream=stream):
            for _ in range(R):
                step()
    reps = max(1, args.steps // R)
    steps = reps * R
    warm_reps = max(1, -(-args.warmup // R))
    gpu_uuid = None
    try:
        gpu_uuid = torch.cuda.get_device_properties(dev).uuid
        gpu_uuid = "GPU-" + str(gpu_uuid) if not str(gpu_uuid).startswith("GPU-") else str(gpu_uuid)
    except Exception:
        gpu_uuid = str(local)
    clocks = ClockSampler(gpu_uuid)

    with torch.cuda.stream(stream):
        for _ in range(warm_reps):
            g_plain.replay()
        stream.synchronize()
        dist_barrier(world)
        torch.cuda.synchronize()
        clocks.start()
        time.sleep(0.3)
        t_wall0 = time.time()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g_plain.replay()
        e1.record(stream)
        e1.synchronize()
        t_wall1 = time.time()
        torch.cuda.synchronize()
        dist_barrier(world)
        clocks.stop()
        # per-kernel breakdown: the same R steps captured with external event-record nodes
        # between the kernels; the graph is replayed, and the last replay's R samples are read
        nb = R
        ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(nb)]
        g_ev = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_ev, stream=stream):
            for b in range(nb):
                step(ev[b])
        ev_reps = max(2, min(reps, 100))
        k0, k1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k0.record(stream)
        for _ in range(ev_reps):
            g_ev.replay()
        k1.record(stream)
        k1.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK, "a kernel reported a timeout"

    ms_total = e0.elapsed_time(e1)
    ms_total = dist_max(ms_total, world)
    ms_step = ms_total / steps
    weights_per_step = sum(d["N"] * d["K"] for d in L)
    value = weak_scaling_value(weights_per_step, steps, ms_total, world)
    # per-kernel breakdown: each kernel group (its launches for all layers) between two events
    per = {k: [] for k in kernels}
    for r in range(nb):
        for ki, k in enumerate(kernels):
            per[k].append(ev[r][ki].elapsed_time(ev[r][ki + 1]))
    peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))) if os.path.exists(
        os.path.join(ROOT, "MEASURED_PEAKS.json")) else {}
    hbm_peak = float(peaks.get("hbm_gbs", 6650.0))
    tc_peak = float(peaks.get("bf16_tflops", 1590.0))
    peak_src = "of measured" if peaks else "of fallback"
    breakdown = {}
    for k in kernels:
        group_ms = float(np.mean(per[k]))           # all layers' launches of this kernel, one step
        if k == "act_scale":
            work = sum(bytes_act_scale(M, d["K"]) for d in L)
        elif k == "quantize":
            work = sum(bytes_quantize(d["N"], d["K"]) for d in L)
        else:
            work = sum(bytes_linear(M, d["N"], d["K"]) for d in L)
        gbs = work / (group_ms * 1e-3) / 1e9
        entry = {"launches_per_step": len(L), "avg_us": 1e3 * group_ms / len(L), "share_of_step": None,
                 "algorithmic_GBps": gbs, "frac_hbm": gbs / hbm_peak}
        if k in ("gemv", "gemm"):
            entry["effective_weight_GBps"] = sum(2 * d["N"] * d["K"] for d in L) / (group_ms * 1e-3) / 1e9
            entry["TFLOPs"] = sum(flops_linear(M, d["N"], d["K"]) for d in L) / (group_ms * 1e-3) / 1e12
            entry["frac_tensor"] = entry["TFLOPs"] / tc_peak
        breakdown[k] = entry
    step_sum_us = sum(e["avg_us"] * e["launches_per_step"] for e in breakdown.values())
    for e in breakdown.values():
        e["share_of_step"] = e["avg_us"] * e["launches_per_step"] / step_sum_us

    dom = max(breakdown, key=lambda k: breakdown[k]["avg_us"] * breakdown[k]["launches_per_step"])
    kfile = {"act_scale": "awq_act.cuh", "quantize": "awq_quant.cuh", "gemv": "awq_gemv.cuh",
             "gemm": "awq_gemm.cuh"}[dom]
    tr = profile_traffic(kfile, wl.name, M)
    if dom == "gemm" and not decode:
        roof = {"bound": "tensor", "achieved": breakdown[dom]["TFLOPs"], "peak": tc_peak, "unit": "TFLOP/s",
                "frac": breakdown[dom]["TFLOPs"] / tc_peak, "traffic": tr["bytes_per_launch"] if tr else None,
                "kernel": dom, "peak_source": peak_src + " (bf16 burst; fp16 dense has the same nominal rate)"}
    else:
        roof = {"bound": "hbm", "achieved": breakdown[dom]["algorithmic_GBps"], "peak": hbm_peak, "unit": "GB/s",
                "frac": breakdown[dom]["algorithmic_GBps"] / hbm_peak,
                "traffic": tr["bytes_per_launch"] if tr else None, "kernel": dom,
                "peak_source": peak_src + " (HBM copy)",
                "algorithmic_bytes_per_launch": {
                    "act_scale": "6*M*K + 4*K", "quantize": "2*N*K + 4*K + packed(N,K)",
                    "gemv": "packed(N,K) + 2*M*K + 2*M*N"}[dom],
                "note": "achieved = algorithmic bytes of the kernel's launches in one step / their summed duration"}

    # ---------------------------------------------------------------- end to end (host buffers, public API)
    e2e = None
    if not args.no_e2e:
        pin = [(torch.from_numpy(x).pin_memory(), torch.from_numpy(W).pin_memory()) for (x, W) in host]
        y_host = [torch.empty((M, d["N"]), dtype=torch.float16).pin_memory() for d in L]
        h2d = sum(x.numel() * 2 + W.numel() * 2 for x, W in pin)
        d2h = sum(y.numel() * 2 for y in y_host)

        def e2e_step():
            for (xh, Wh), d, yh in zip(pin, L, y_host):
                d["x"].copy_(xh, non_blocking=True)
                d["W"].copy_(Wh, non_blocking=True)
                P.awq_activation_scale(d["x"], 0.5, d["s"], d["xs"])
                P.awq_quantize_g128(d["W"], d["s"], d["packed"])
                lin(d["xs"], *d["packed"], d["N"], d["y"])
                yh.copy_(d["y"], non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(3):
                e2e_step()
            stream.synchronize()
            dist_barrier(world)
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            for _ in range(args.e2e_steps):
                e2e_step()
            a1.record(stream)
            a1.synchronize()
        ms_e2e = dist_max(a0.elapsed_time(a1), world)
        e2e = {"value": weak_scaling_value(weights_per_step, args.e2e_steps, ms_e2e, world), "unit": "GB/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps,
               "note": "pinned host x and W copied in, y copied out, every step, through the Python binding"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(host)

    launches = steps * len(L) * len(kernels)
    line = {
        "metric": metric_name(M), "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": warm_reps * R, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": bench_config(wl, M), "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks.summary(t_wall0, t_wall1), "breakdown": breakdown,
        "breakdown_method": ("graph of %d steps, each with external CUDA event-record nodes around its "
                             "a1 / a2 / linear kernel groups, replayed %d times; the last replay's samples "
                             "are averaged" % (nb, ev_reps)),
        "ms_per_step_with_kernel_events": k0.elapsed_time(k1) / (ev_reps * nb),
        "timing": "CUDA events around %d replays of a captured graph of %d steps; inputs larger than L2" % (reps, R),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g_plain, g_ev
    dist_done(world)


def main():
    args = parse_args()
    world, rank, local = dist_init(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
