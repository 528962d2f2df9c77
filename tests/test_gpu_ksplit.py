"""GPU parity of the prefill kernel's K split (a CTA pair per output tile, each over half of K,
rank 1's fp32 partial sums pushed into rank 0's shared memory) against the oracle.

awq_debug_set_gemm_split forces the split off (1), on for every tile (2), or the mixed form (3:
whole rounds of one tile per CTA, then the remaining tiles split, on a grid of 3 CTA pairs so
that small layers take both kinds of work item). Every form runs on the same shapes, token tiles
32 to 256, every epilogue, and K from one group pair upward; the split forms must be
deterministic and within the same bars as the unsplit one.
"""
import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads
from gpu_util import assert_tight, assert_tolerance, dev, f16_bits, host, lib, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib()


@pytest.fixture
def split():
    P = lib()
    yield P.awq_debug_set_gemm_split
    P.awq_debug_set_gemm_split(0)


def _prep(x, W):
    P = lib()
    s, xs = P.awq_activation_scale(dev(x), 0.5)
    return xs, P.awq_quantize_g128(dev(W), s)


# M picks the token tile (32, 64, then the round model's 64/128/256); K = 128 gives each CTA of
# the pair a single 64-k step.
@pytest.mark.parametrize("M", [5, 33, 100, 300, 513])
@pytest.mark.parametrize("N,K", [(256, 128), (200, 384), (1000, 1280), (136, 2304), (896, 640)])
def test_split_matches_oracle_and_unsplit(split, M, N, K):
    P = lib()
    x, W = workloads.random_case(211 + M, M, N, K)
    r = O.reference_forward(x, W)
    xs, pk = _prep(x, W)
    out = {}
    for ks in (1, 2, 3):
        split(ks)
        y = host(P.awq_w4a16_gemm(xs, *pk, N))
        assert P.awq_poll_device_status() == P.AWQ_OK
        assert_tolerance(y.astype(np.float64), r["y"], f"gemm ks={ks} M={M} N={N} K={K}")
        assert_tight(y, r["y"], rel=2.0 ** -10, abs_rms=3e-3, what=f"gemm ks={ks}")
        out[ks] = y
    for ks in (2, 3):
        split(ks)
        again = host(P.awq_w4a16_gemm(xs, *pk, N))
        assert np.array_equal(f16_bits(again), f16_bits(out[ks])), f"split form {ks} not deterministic"


@pytest.mark.parametrize("ks", [2, 3])
@pytest.mark.parametrize("M", [40, 300])
def test_split_fused_epilogues(split, M, ks):
    P = lib()
    split(ks)
    Nq, Nkv, K = 512, 128, 1280
    x, W = workloads.random_case(231 + M, M, Nq + 2 * Nkv, K)
    r = O.reference_forward(x, W)
    xs, pk = _prep(x, W)
    q, k, v = P.awq_w4a16_linear_qkv(xs, *pk, Nq, Nkv)
    for got, ref, name in zip((q, k, v), O.split_qkv(r["y"], Nq, Nkv), "qkv"):
        assert_tolerance(host(got).astype(np.float64), ref, f"split {name} M={M}")
    I = 1008
    x2, W2 = workloads.random_case(241 + M, M, 2 * I, K)
    r2 = O.reference_forward(x2, W2)
    xs2, pk2 = _prep(x2, W2)
    h = host(P.awq_w4a16_linear_silu_mul(xs2, *pk2, I)).astype(np.float64)
    h_ref = O.gate_up_silu(r2["y"])
    ef = np.linalg.norm(h - h_ref) / np.linalg.norm(h_ref)
    assert ef <= 2e-3, f"split silu*up M={M}: rel Frobenius {ef:.3e}"
    assert P.awq_poll_device_status() == P.AWQ_OK


def test_split_full_size_down_proj_sampled(split):
    """Llama-3-8B down_proj (4096 x 14336) at M = 512, split forced on: sampled outputs."""
    P = lib()
    split(2)
    wl = workloads.WORKLOADS["llama3_8b_prefill"]
    M = 512
    x, W = workloads.layer_inputs(wl, 3, M)
    N = W.shape[0]
    xs, pk = _prep(x, W)
    y = host(P.awq_w4a16_gemm(xs, *pk, N))
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, 160, replace=False)]))
    toks = np.unique(np.concatenate([[0, M - 1], rng.choice(M, 16, replace=False)]))
    s = O.activation_scale(x)
    y_ref = O.linear(O.scale_activations(x[toks], s), O.dequantize(*O.quantize_groups(O.fold_weights(W[rows], s))))
    assert_tolerance(y[np.ix_(toks, rows)].astype(np.float64), y_ref, "split down_proj sampled")


def test_split_hook_rejects_bad_values():
    P = lib()
    for bad in (-1, 4):
        assert P.load_library().awq_debug_set_gemm_split(bad) == P.AWQ_ERR_INVALID_ARG
