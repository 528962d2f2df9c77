"""GPU parity of the quantizer variants (INT3-g128, symmetric INT4/INT3) and of the linear
kernels on their packed weights, against the oracle's quantize_groups_cfg.

The codes, scales and zero points are compared bit for bit with the oracle's packing; the
layer outputs (decode and prefill kernels, which dequantize every variant as (q - z) S) within
the bar of the linear tests.
"""
import json
import os

import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads
from gpu_util import assert_tolerance, dev, f16_bits, host, lib, torch_mod

pytestmark = pytest.mark.gpu

VARIANTS = [(4, False), (3, True), (3, False)]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib()


def _oracle_packed(W, s, bits, zero_point):
    wf = O.fold_weights(W, s) if s is not None else np.asarray(W, np.float16)
    q, S, z = O.quantize_groups_cfg(wf, bits, 128, zero_point)
    return O.pack(q, S, z), (q, S, z)


def _variant_check(W, s, bits, zero_point):
    P = lib()
    ref, _ = _oracle_packed(W, s, bits, zero_point)
    qw, sc, zb = P.awq_quantize(dev(W), dev(s) if s is not None else None, bits=bits, zero_point=zero_point)
    assert np.array_equal(host(qw).view(np.uint32), ref[0]), "codes"
    assert np.array_equal(f16_bits(host(sc)), f16_bits(ref[1])), "scales"
    assert np.array_equal(host(zb), ref[2]), "zeros"
    return qw, sc, zb


@pytest.mark.parametrize("bits,zero_point", VARIANTS)
@pytest.mark.parametrize("N,K,fold", [(128, 128, False), (200, 384, True), (77, 640, True), (1000, 1280, False),
                                      (300, 11008, True)])
def test_variant_quantize_bit_exact(bits, zero_point, N, K, fold):
    x, W = workloads.random_case(31 + bits, 4, N, K)
    s = O.activation_scale(x) if fold else None
    _variant_check(W, s, bits, zero_point)


@pytest.mark.parametrize("bits,zero_point", VARIANTS)
def test_variant_quantize_hand_groups_and_extremes(bits, zero_point):
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quantizer_variant_cases.json")))
    rows = [list(c["values"]) + [c["fill"]] * (128 - len(c["values"])) for c in fx["groups"]]
    rng = np.random.default_rng(4)
    rows.append(list(np.where(rng.random(128) < 0.5, 65504.0, -65504.0)))     # full fp16 range
    rows.append([6e-8 * (i % 3) for i in range(128)])                          # subnormals
    rows.append([float(v) for v in rng.uniform(0.5, 1.5, 128)])                # all positive
    rows.append([float(v) for v in -rng.uniform(0.5, 1.5, 128)])               # all negative
    W = np.array(rows * 3, dtype=np.float16)
    W = np.concatenate([W, W[:, ::-1]], axis=1)
    _variant_check(W, None, bits, zero_point)
    s = np.ones(256, np.float32)
    s[:8] = 4096.0        # overflow to inf after the fold
    s[8:16] = 1e-3
    _variant_check(W, s, bits, zero_point)


def test_variant_golden_cases_on_the_gpu():
    """The hand-derived groups give their hand-derived codes, scales and zeros on the GPU too."""
    P = lib()
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quantizer_variant_cases.json")))
    for c in fx["groups"]:
        vals = list(c["values"]) + [c["fill"]] * (128 - len(c["values"]))
        W = np.array([vals] * 16, dtype=np.float16)                      # one full 16-row tile
        qw, sc, zb = P.awq_quantize(dev(W), None, bits=c["bits"], zero_point=c["zero_point"])
        q, S, z = O.unpack(host(qw).view(np.uint32), host(sc), host(zb), 16, 128)
        expect = list(c["codes"]) + [c["fill_code"]] * (128 - len(c["codes"]))
        assert q[0].tolist() == expect, c["name"]
        assert int(f16_bits(S)[0, 0]) == int(c["scale_bits"], 16), c["name"]
        assert int(z[0, 0]) == c["zero"], c["name"]


@pytest.mark.parametrize("bits,zero_point", VARIANTS)
def test_variant_full_size_layer_bit_exact(bits, zero_point):
    """A full Llama-2-7B down_proj layer (4096 x 11008) with the AWQ fold."""
    wl = workloads.WORKLOADS["llama2_7b_decode_m1"]
    x, W = workloads.layer_inputs(wl, 3, 1)
    _variant_check(W, O.activation_scale(x), bits, zero_point)


@pytest.mark.parametrize("bits,zero_point", VARIANTS)
@pytest.mark.parametrize("M,N,K", [(1, 512, 1024), (5, 300, 640), (64, 200, 1280), (300, 256, 512)])
def test_variant_linear_matches_oracle(bits, zero_point, M, N, K):
    """Decode (M <= 32) and prefill kernels on variant weights against the oracle's dequantized product."""
    P = lib()
    x, W = workloads.random_case(41 + bits, M, N, K)
    s = O.activation_scale(x)
    xs = O.scale_activations(x, s)
    _, (q, S, z) = _oracle_packed(W, s, bits, zero_point)
    y_ref = O.linear(xs, O.dequantize_cfg(q, S, z, 128))
    packed = P.awq_quantize(dev(W), dev(s), bits=bits, zero_point=zero_point)
    y = P.awq_w4a16_linear(dev(xs), *packed, N)
    assert P.awq_poll_device_status() == P.AWQ_OK
    assert_tolerance(host(y).astype(np.float64), y_ref, f"linear bits={bits} zp={zero_point} M={M}")
    if M <= 32:
        y2 = P.awq_w4a16_gemm(dev(xs), *packed, N)
        assert_tolerance(host(y2).astype(np.float64), y_ref, f"prefill kernel bits={bits} zp={zero_point} M={M}")
