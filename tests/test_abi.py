"""The C-ABI library: it builds, loads and exports every declared symbol; host-only logic.

No test here calls into CUDA: argument checks that fail return before the
library touches the device, and only those paths are exercised.
"""
import ctypes
import json
import os
import re
import subprocess

import pytest

from oracle import awq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "awq_w4a16.h")


@pytest.fixture(scope="module")
def lib():
    from weight_only_quantization_w4a16_b200 import build as B
    import weight_only_quantization_w4a16_b200 as P
    B.build()
    return P.load_library()


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"^AWQ_API [^(]*?\b(awq_\w+)\(", src, flags=re.M)))


def test_header_declares_the_path():
    names = _declared()
    for n in ["awq_activation_scale", "awq_scale_activations", "awq_quantize_g128", "awq_w4a16_gemv",
              "awq_w4a16_gemm", "awq_w4a16_linear", "awq_poll_device_status", "awq_layout_version",
              "awq_search_alpha", "awq_search_workspace_bytes"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    import weight_only_quantization_w4a16_b200 as P
    out = subprocess.run(["nm", "-D", "--defined-only", P.library_path()], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (awq_\w+)$", out, flags=re.M))
    declared = set(_declared())
    assert declared <= exported, declared - exported
    # nothing else leaks out of the library (static cudart stays internal)
    assert all(name.startswith("awq_") for name in re.findall(r" [TDBRW] (\S+)$", out, flags=re.M))
    for name in declared:
        assert hasattr(lib, name)


def test_debug_bounds_library_exports_the_same_symbols():
    """The -DAWQ_DEBUG_BOUNDS build (built by build(); the GPU tests run it) has the same ABI."""
    from weight_only_quantization_w4a16_b200 import build as B
    path = B.build(debug_bounds=True)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (awq_\w+)$", out, flags=re.M))
    assert set(_declared()) <= exported
    dbg = ctypes.CDLL(path)
    assert dbg.awq_layout_version() == 2


def test_layout_version_and_status_strings(lib):
    assert lib.awq_layout_version() == 2
    for code in range(7):
        s = lib.awq_status_string(code).decode()
        assert s.startswith("AWQ_")
    assert lib.awq_status_string(99).decode() == "AWQ_ERR_UNKNOWN"


def test_check_config_against_page_configs(lib):
    fx = json.load(open(os.path.join(ROOT, "tests", "golden", "quant_configs.json")))
    hf = fx["hf_quantization_config"]
    assert lib.awq_check_config(hf["bits"], hf["group_size"], int(hf["zero_point"])) == 0
    aw = fx["autoawq_quant_config"]
    assert lib.awq_check_config(aw["w_bit"], aw["q_group_size"], int(aw["zero_point"])) == 0
    for v in fx["supported_variants"]:
        assert lib.awq_check_config(v["bits"], v["group_size"], int(v["zero_point"])) == 0
    for u in fx["unsupported_examples"]:
        assert lib.awq_check_config(u["bits"], u["group_size"], int(u["zero_point"])) == 2


def test_gemm_split_hook_is_host_only(lib):
    """The K-split test hook takes 0, 1 or 2 and touches no device."""
    for bad in (-1, 4, 100):
        assert lib.awq_debug_set_gemm_split(bad) == 1
    for ok in (3, 2, 1, 0):
        assert lib.awq_debug_set_gemm_split(ok) == 0


# The prefill kernel's launch plan on 148 SMs for the Llama-3-8B prefill layers: each entry is
# the fastest form, or within 5% of it, in per-layer sweeps that forced every token tile with the
# K split off, on for every tile, and on for the last round's tiles only (CUDA events, B200).
PLAN_CASES = [
    # (M, N, K, token tile, K split, split tiles)
    (512, 6144, 4096, 256, 1, 0),       # q/k/v: 96 tiles, a split would add a round
    (512, 4096, 4096, 256, 2, 64),      # o_proj: 64 tiles, all split
    (512, 28672, 4096, 256, 2, 4),      # gate/up: 3 whole rounds of 148 tiles, the last 4 split
    (512, 4096, 14336, 256, 2, 64),     # down_proj: 64 tiles, all split
    (128, 6144, 4096, 128, 2, 48),
    (128, 4096, 4096, 64, 2, 64),
    (128, 28672, 4096, 128, 1, 0),
    (128, 4096, 14336, 64, 2, 64),
    (2048, 28672, 4096, 256, 1, 0),     # 12.1 rounds: splitting the last 16 tiles measured no gain
    (2048, 6144, 4096, 256, 1, 0),      # 384 tiles: 88 left over, more than 74 pairs
    (32, 4096, 4096, 32, 2, 32),
    (512, 28672, 8192, 256, 2, 4),      # Llama-2-70B gate/up: 234.5 us against 256.7 without the split
    (512, 8192, 28672, 256, 1, 0),      # Llama-2-70B down: 128 tiles, one round
]


@pytest.mark.parametrize("M,N,K,bt,ks,nsplit", PLAN_CASES)
def test_gemm_plan_matches_measured_choices(lib, M, N, K, bt, ks, nsplit):
    import weight_only_quantization_w4a16_b200 as P
    assert P.awq_gemm_plan(M, N, K, 0, num_sms=148) == (bt, ks, nsplit)


def test_gemm_plan_hook_and_argument_checks(lib):
    import weight_only_quantization_w4a16_b200 as P
    try:
        P.awq_debug_set_gemm_split(1)
        assert P.awq_gemm_plan(512, 4096, 14336, 0, num_sms=148)[1:] == (1, 0)
        P.awq_debug_set_gemm_split(2)
        assert P.awq_gemm_plan(2048, 28672, 4096, 0, num_sms=148)[1:] == (2, 224 * 8)
        # form 3 (3 CTA pairs): the GPU tests' shape 300 x 1000 x 1280 takes whole-tile rounds and
        # split tiles in one launch
        P.awq_debug_set_gemm_split(3)
        bt, ks, nsplit = P.awq_gemm_plan(300, 1000, 1280, 0, num_sms=148)
        assert ks == 2 and 0 < nsplit < 8 * -(-300 // bt)
    finally:
        P.awq_debug_set_gemm_split(0)
    bt, ks, ns = ctypes.c_int(), ctypes.c_int(), ctypes.c_longlong()
    ref = (ctypes.byref(bt), ctypes.byref(ks), ctypes.byref(ns))
    assert lib.awq_gemm_plan(0, 16, 128, 0, 148, *ref) == 1
    assert lib.awq_gemm_plan(1, 16, 100, 0, 148, *ref) == 1
    assert lib.awq_gemm_plan(1, 16, 128, 3, 148, *ref) == 1
    assert lib.awq_gemm_plan(1, 16, 128, 0, 0, *ref) == 1
    assert lib.awq_gemm_plan(1, 48, 128, 2, 148, *ref) == 1       # SiLU: N = 2 I, I % 16 == 0
    assert lib.awq_gemm_plan(1, 16, 128, 0, 148, None, None, None) == 1
    assert lib.awq_gemm_plan(64, 64, 128, 2, 148, *ref) == 0 and (bt.value, ks.value, ns.value) == (64, 2, 1)


def test_quantize_variant_argument_checks(lib):
    """awq_quantize rejects unbuilt configurations before any CUDA call (no GPU needed)."""
    V = ctypes.c_void_p
    for bits, group, zp in ((4, 64, 1), (8, 128, 1), (3, 64, 0)):
        assert lib.awq_quantize(V(0x10000), None, 16, 256, bits, group, zp, V(0x10000), V(0x10000), V(0x10000), None) == 2
    assert lib.awq_quantize(None, None, 16, 256, 3, 128, 0, V(0x10000), V(0x10000), V(0x10000), None) == 1


@pytest.mark.parametrize("N,K", [(1, 128), (128, 128), (300, 256), (4096, 11008), (28672, 8192), (513, 640)])
def test_packed_sizes_match_layout_spec(lib, N, K):
    words, sc, zb = O.packed_sizes(N, K)
    assert lib.awq_qweight_bytes(N, K) == 4 * words
    assert lib.awq_scales_bytes(N, K) == 2 * sc
    assert lib.awq_zeros_bytes(N, K) == zb


@pytest.mark.parametrize("N,K", [(0, 128), (16, 0), (16, 100), (16, 192), (-1, 128), (2147483647, 128),
                                 (2147483521, 128), (2 ** 30, 256)])
def test_packed_sizes_reject_bad_shapes(lib, N, K):
    assert lib.awq_qweight_bytes(N, K) == 0 and lib.awq_scales_bytes(N, K) == 0 and lib.awq_zeros_bytes(N, K) == 0


A = 0x10000   # aligned fake addresses: never dereferenced, every call below fails its checks first
MIS = 0x10008


def test_argument_checks_fail_before_any_device_call(lib):
    V = ctypes.c_void_p
    # null pointers
    assert lib.awq_quantize_g128(None, None, 16, 128, V(A), V(A), V(A), None) == 1
    assert lib.awq_w4a16_gemv(V(A), V(A), V(A), None, V(A), 1, 16, 128, None) == 1
    assert lib.awq_w4a16_gemm(None, V(A), V(A), V(A), V(A), 1, 16, 128, None) == 1
    assert lib.awq_activation_scale(None, 1, 128, 0.5, V(A), None, None) == 1
    assert lib.awq_scale_activations(V(A), None, 1, 128, V(A), None) == 1
    # bad sizes
    assert lib.awq_quantize_g128(V(A), None, 16, 100, V(A), V(A), V(A), None) == 1
    assert lib.awq_quantize_g128(V(A), None, 0, 128, V(A), V(A), V(A), None) == 1
    assert lib.awq_w4a16_gemv(V(A), V(A), V(A), V(A), V(A), 33, 16, 128, None) == 1
    assert lib.awq_w4a16_gemv(V(A), V(A), V(A), V(A), V(A), 0, 16, 128, None) == 1
    assert lib.awq_w4a16_gemm(V(A), V(A), V(A), V(A), V(A), 4, 16, 192, None) == 1
    assert lib.awq_activation_scale(V(A), 1, 12, 0.5, V(A), None, None) == 1
    assert lib.awq_activation_scale(V(A), 1, 128, float("nan"), V(A), None, None) == 1
    # row counts whose padding would overflow an int, and layers past 2^34 packed weights
    assert lib.awq_w4a16_gemv(V(A), V(A), V(A), V(A), V(A), 1, 2147483647, 128, None) == 1
    assert lib.awq_w4a16_gemm(V(A), V(A), V(A), V(A), V(A), 64, 2147483600, 128, None) == 1
    assert lib.awq_quantize_g128(V(A), None, 2147483647, 128, V(A), V(A), V(A), None) == 1
    assert lib.awq_w4a16_linear(V(A), V(A), V(A), V(A), V(A), 1, 2 ** 27, 256, None) == 1
    # the scale search: bad shapes, null outputs, a short workspace, a non-finite candidate
    a1 = (ctypes.c_float * 1)(0.5)
    anan = (ctypes.c_float * 1)(float("nan"))
    assert lib.awq_search_workspace_bytes(0, 16, 128) == 0 and lib.awq_search_workspace_bytes(4, 16, 100) == 0
    need = lib.awq_search_workspace_bytes(4, 16, 128)
    assert need > 0
    assert lib.awq_search_alpha(V(A), V(A), 4, 16, 128, a1, 1, None, V(A), V(A), need, None) == 1
    assert lib.awq_search_alpha(V(A), V(A), 4, 16, 128, a1, 1, V(A), V(A), V(A), need - 1, None) == 1
    assert lib.awq_search_alpha(V(A), V(A), 4, 16, 128, anan, 1, V(A), V(A), V(A), need, None) == 1
    assert lib.awq_search_alpha(V(A), V(A), 4, 16, 128, a1, 0, V(A), V(A), V(A), need, None) == 1
    assert lib.awq_search_alpha(V(MIS), V(A), 4, 16, 128, a1, 1, V(A), V(A), V(A), need, None) == 3
    # fused epilogues: I a positive multiple of 16, Nq and Nkv positive, aligned outputs
    assert lib.awq_w4a16_linear_silu_mul(V(A), V(A), V(A), V(A), V(A), 1, 24, 128, None) == 1
    assert lib.awq_w4a16_linear_silu_mul(V(A), V(A), V(A), V(A), V(A), 1, 0, 128, None) == 1
    assert lib.awq_w4a16_linear_qkv(V(A), V(A), V(A), V(A), V(A), V(A), V(A), 1, 64, 0, 128, None) == 1
    assert lib.awq_w4a16_linear_qkv(V(A), V(A), V(A), V(A), V(A), V(A), None, 1, 64, 8, 128, None) == 1
    assert lib.awq_w4a16_linear_qkv(V(A), V(A), V(A), V(A), V(A), V(MIS), V(A), 1, 64, 8, 128, None) == 3
    # misaligned pointers
    assert lib.awq_quantize_g128(V(MIS), None, 16, 128, V(A), V(A), V(A), None) == 3
    assert lib.awq_w4a16_gemv(V(A), V(A), V(A), V(A), V(MIS), 1, 16, 128, None) == 3
    assert lib.awq_w4a16_gemm(V(A), V(MIS), V(A), V(A), V(A), 300, 16, 128, None) == 3
    assert lib.awq_scale_activations(V(A), V(MIS), 1, 128, V(A), None) == 3


def test_binding_refuses_to_run_without_library(tmp_path):
    import weight_only_quantization_w4a16_b200 as P
    with pytest.raises(RuntimeError, match="no fallback"):
        P.load_library(str(tmp_path / "missing.so"))
