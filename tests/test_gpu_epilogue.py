"""GPU parity of the fused-module epilogues ("transformers - AWQ" section 3) against the oracle.

The whole path runs on the GPU (activation statistic, fold + quantizer, the fused linear
call); the oracle computes the plain layer in float64 and applies its own split_qkv or
gate_up_silu. Decode (M <= 32, the ring decode kernel) and prefill (tcgen05) paths.
"""
import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads
from gpu_util import assert_tolerance, dev, host, lib, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib()


def assert_silu_tolerance(h, y_ref, what):
    """The linear layer's bar, propagated through h = SiLU(g) * u.

    The stated bar bounds each linear output: |dy| <= 1e-2 rms(y_ref). Through h it allows
    |dh| <= (|SiLU'(g)| |u| + |SiLU(g)|) 1e-2 rms(y_ref) per element (first order), with
    SiLU'(g) = sig(g) (1 + g (1 - sig(g))). The relative Frobenius bar 2e-3 applies to h as it is."""
    I = y_ref.shape[1] // 2
    g, u = y_ref[:, :I], y_ref[:, I:]
    h_ref = O.gate_up_silu(y_ref)
    sig = 1.0 / (1.0 + np.exp(-g))
    dsilu = sig * (1.0 + g * (1.0 - sig))
    rms = np.sqrt(np.mean(y_ref ** 2))
    bound = (np.abs(dsilu) * np.abs(u) + np.abs(O.silu(g))) * 1e-2 * rms
    err = np.abs(np.asarray(h, np.float64) - h_ref)
    ef = np.linalg.norm(err) / np.linalg.norm(h_ref)
    assert ef <= 2e-3, f"{what}: rel Frobenius {ef:.3e} (bar 2e-3)"
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond the propagated bar; worst {np.max(err - bound):.3e}"


def _prep(x, W):
    P = lib()
    s, xs = P.awq_activation_scale(dev(x), 0.5)
    return xs, P.awq_quantize_g128(dev(W), s)


@pytest.mark.parametrize("M", [1, 2, 5, 17, 32, 64, 300])
@pytest.mark.parametrize("Nq,Nkv,K", [(512, 128, 512), (200, 24, 384)])
def test_qkv_split(M, Nq, Nkv, K):
    P = lib()
    x, W = workloads.random_case(131 + M, M, Nq + 2 * Nkv, K)
    r = O.reference_forward(x, W)
    xs, pk = _prep(x, W)
    q, k, v = P.awq_w4a16_linear_qkv(xs, *pk, Nq, Nkv)
    for got, ref, name in zip((q, k, v), O.split_qkv(r["y"], Nq, Nkv), "qkv"):
        assert_tolerance(host(got).astype(np.float64), ref, f"{name} M={M}")


@pytest.mark.parametrize("M", [1, 2, 5, 17, 32, 64, 300])
@pytest.mark.parametrize("I,K", [(256, 512), (1008, 384), (48, 1280)])
def test_gate_up_silu(M, I, K):
    P = lib()
    x, W = workloads.random_case(141 + M, M, 2 * I, K)
    r = O.reference_forward(x, W)
    xs, pk = _prep(x, W)
    h = P.awq_w4a16_linear_silu_mul(xs, *pk, I)
    assert_silu_tolerance(host(h), r["y"], f"silu*up M={M} I={I}")


@pytest.mark.parametrize("M", [1, 512])
def test_llama_shapes_sampled(M):
    """Llama-3-8B q/k/v (4096 + 2 x 1024 rows) and Llama-2-7B gate+up (2 x 11008 rows), full size."""
    P = lib()
    wl = workloads.WORKLOADS["llama3_8b_prefill"]
    x, W = workloads.layer_inputs(wl, 0, M)
    xs, pk = _prep(x, W)
    q, k, v = P.awq_w4a16_linear_qkv(xs, *pk, 4096, 1024)
    rows = np.array([0, 1, 777, 4095, 4096, 4500, 5119, 5120, 6000, 6143])
    toks = np.unique(np.array([0, M - 1, M // 2]))
    wf = O.fold_weights(W[rows], O.activation_scale(x))
    y_ref = O.linear(O.scale_activations(x, O.activation_scale(x))[toks], O.dequantize(*O.quantize_groups(wf)))
    got = np.concatenate([host(q), host(k), host(v)], axis=1)[np.ix_(toks, rows)]
    assert_tolerance(got.astype(np.float64), y_ref, "llama3 qkv sampled")

    wl2 = workloads.WORKLOADS["llama2_7b_decode_m1"]
    x2, W2 = workloads.layer_inputs(wl2, 2, 1)
    x2 = np.repeat(x2, M, axis=0) if M > 1 else x2
    xs2, pk2 = _prep(x2, W2)
    h = host(P.awq_w4a16_linear_silu_mul(xs2, *pk2, 11008))
    idx = np.array([0, 5, 4096, 11007])
    s2 = O.activation_scale(x2)
    wf2 = O.fold_weights(np.concatenate([W2[idx], W2[11008 + idx]]), s2)
    y2 = O.linear(O.scale_activations(x2, s2)[:1], O.dequantize(*O.quantize_groups(wf2)))
    assert_silu_tolerance(h[:1, idx], y2, "llama2 gate/up sampled")
