"""The bounds-checking build (libawq_w4a16_debug_bounds.so, compiled with -DAWQ_DEBUG_BOUNDS) on
small ragged cases of every kernel: no index check fires (awq_poll_device_status stays AWQ_OK)
and every output equals the normal build's bit for bit.

The checks stand in for a memory checker on this hardware: they compare the kernels' computed
offsets (ring slots, packed-array ranges, record indices, cluster pushes) with the extents of the
buffers they address, and skip the access when one is out of range.
"""
import numpy as np
import pytest

import workloads
from oracle import awq_oracle as O
from gpu_util import dev, host, lib, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    P = lib()
    from weight_only_quantization_w4a16_b200 import build as B
    path = B.build(debug_bounds=True)
    return P, P.load_library(), P.load_library(path)


def _both(P, rel, dbg, fn):
    """fn() once through each library; returns (release outputs, debug outputs) as numpy arrays."""
    saved = P._lib
    try:
        P._lib = rel
        a = fn()
        P._lib = dbg
        b = fn()
        assert P.awq_poll_device_status() == P.AWQ_OK, "a bounds check fired"
    finally:
        P._lib = saved
    as_np = lambda t: [host(v) for v in (t if isinstance(t, (tuple, list)) else (t,))]
    return as_np(a), as_np(b)


def _same(a, b, what):
    for x, y in zip(a, b):
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8)), what


@pytest.mark.parametrize("M,N,K", [(1, 200, 640), (5, 77, 384), (20, 300, 1280), (32, 130, 256), (64, 200, 640),
                                   (300, 144, 512)])
def test_linear_path_under_bounds_checks(libs, M, N, K):
    P, rel, dbg = libs
    x, W = workloads.random_case(61, M, N, K)
    xd, Wd = dev(x), dev(W)

    def run():
        s, xs = P.awq_activation_scale(xd, 0.5)
        packed = P.awq_quantize_g128(Wd, s)
        y = P.awq_w4a16_linear(xs, *packed, N)
        return (s, xs, *packed, y)
    a, b = _both(P, rel, dbg, run)
    _same(a, b, f"linear path M={M} N={N} K={K}")
    if M <= 32:
        a, b = _both(P, rel, dbg, lambda: P.awq_w4a16_gemm(dev(O.scale_activations(x, O.activation_scale(x))),
                                                            *P.awq_quantize_g128(Wd, dev(O.activation_scale(x))), N))
        _same(a, b, "prefill kernel at small M")


@pytest.mark.parametrize("bits,zero_point", [(4, False), (3, True), (3, False)])
def test_quantizer_variants_under_bounds_checks(libs, bits, zero_point):
    P, rel, dbg = libs
    x, W = workloads.random_case(62, 4, 77, 640)
    a, b = _both(P, rel, dbg, lambda: P.awq_quantize(dev(W), dev(O.activation_scale(x)), bits=bits,
                                                     zero_point=zero_point))
    _same(a, b, f"quantize bits={bits} zp={zero_point}")


@pytest.mark.parametrize("M", [1, 40])
def test_fused_epilogues_under_bounds_checks(libs, M):
    P, rel, dbg = libs
    nq, nkv, I, K = 256, 64, 176, 512
    x, Wqkv = workloads.random_case(63, M, nq + 2 * nkv, K)
    _, Wgu = workloads.random_case(64, M, 2 * I, K)
    xs = dev(x)
    pq = P.awq_quantize_g128(dev(Wqkv))
    pg = P.awq_quantize_g128(dev(Wgu))
    a, b = _both(P, rel, dbg, lambda: P.awq_w4a16_linear_qkv(xs, *pq, nq, nkv))
    _same(a, b, "q/k/v epilogue")
    a, b = _both(P, rel, dbg, lambda: P.awq_w4a16_linear_silu_mul(xs, *pg, I))
    _same(a, b, "gate/up SiLU epilogue")


def test_search_under_bounds_checks(libs):
    P, rel, dbg = libs
    x, W = workloads.random_case(65, 12, 200, 640)
    a, b = _both(P, rel, dbg, lambda: P.awq_search_alpha(dev(x), dev(W))[:2])
    _same(a, b, "scale search")
