"""Host-side logic of bench.py that decides what the JSON line reports (CPU only)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_code_hash_ignores_comments_and_whitespace_only():
    a = "int f(int x) {\n  return x + 1;  // add one\n}\n"
    b = "/* a header\n   comment */\nint  f(int x){ return x+1; }\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.code_hash(a) == bench.code_hash(b)
    assert bench.code_hash(a) != bench.code_hash(c)


def test_traffic_record_applies_only_to_its_workload_and_unchanged_code():
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    wl, M = d["_workload"], d["_M"]
    assert "awq_gemv.cuh" in d   # the kernel of the default bench step
    for name in ("awq_quant.cuh", "awq_gemv.cuh", "awq_act.cuh"):
        # reported exactly while the recorded code hash matches the kernel code
        e = bench.profile_traffic(name, wl, M)
        if name in d and d[name]["source_sha256_16"] == bench.kernel_source_hash(name):
            assert e is not None and e["bytes_per_step"] > 0
        else:
            assert e is None
        # another workload or M never gets a traffic figure
        assert bench.profile_traffic(name, "llama2_70b_layers", M) is None
        assert bench.profile_traffic(name, wl, M + 1) is None


def test_every_workload_has_a_bench_config():
    import workloads
    for name in workloads.workload_names():
        wl = workloads.WORKLOADS[name]
        for M in wl.Ms:
            cfg = bench.bench_config(wl, M)
            assert cfg["workload"] == name and cfg["M"] == M
            assert ("decode GEMV" in cfg["step"]) == (M <= 32)


def test_exact_step_plan_times_exactly_k_steps():
    for steps in [1, 3, 20, 49, 50, 51, 100, 2000, 2017]:
        R, full, rem = bench.exact_step_plan(steps, 50)
        assert R * full + rem == steps and 0 <= rem < R and R <= 50


def test_rotation_covers_four_times_l2():
    l2 = 126 * 1024 * 1024
    for set_bytes in [8.7e6, 105e6, 122e6, 600e6]:
        n = bench.rotation_sets(int(set_bytes), l2)
        assert n >= 2 and n * set_bytes >= 4 * l2


def test_packed_bytes_matches_the_layout():
    from oracle import awq_oracle as O
    for N, K in [(4096, 4096), (12288, 4096), (4096, 11008), (300, 384), (28672, 8192)]:
        words, halves, zb = O.packed_sizes(N, K)
        assert bench.packed_bytes(N, K) == 4 * words + 2 * halves + zb


def test_parse_defaults_and_reference_metric():
    a = bench.parse_args([])
    assert a.steps > 0 and a.warmup >= 3 and a.impl == "ours" and a.workload == "llama2_7b_decode_m1"
    assert "GEMV" in bench.metric_name(1)
