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
    for name in ("awq_quant.cuh", "awq_gemv.cuh", "awq_act.cuh"):
        # reported exactly while the recorded code hash matches the kernel code
        e = bench.profile_traffic(name, wl, M)
        if d[name]["source_sha256_16"] == bench.kernel_source_hash(name):
            assert e is not None and e["bytes_per_launch"] > 0
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
