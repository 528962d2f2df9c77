"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

* a1 activation statistic and scaling: bit-exact (alpha = 0.5; other alphas
  within one fp32 ulp for s, as the power is not correctly rounded).
* a2 quantizer: packed codes, scales and zeros byte-identical to the oracle's
  codes packed by the oracle's own packer.
* a3 / a4 linear layers: within the bar ||dy||_F / ||y||_F <= 2e-3 and
  max |dy| <= 1e-2 rms(y), plus a tighter bound that the arithmetic allows.

Sizes span several tiles with ragged tails (N not a multiple of 128, M not a
multiple of the token tile, K-slices that do not divide evenly); the full
sizes of the decode and prefill workloads are checked on sampled outputs.
"""
import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads
from gpu_util import (assert_tight, assert_tolerance, dev, f16_bits, host, lib, oracle_packed, torch_mod,
                      upload_packed)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib()
    yield
    torch.cuda.synchronize()


# ----------------------------------------------------------------------------- a1
@pytest.mark.parametrize("M,K", [(1, 512), (7, 384), (32, 2048), (33, 4096), (300, 1280), (1000, 11008), (4096, 512)])
def test_activation_scale_bit_exact(M, K):
    P = lib()
    x, _ = workloads.random_case(11, M, 16, K)
    s, xs = P.awq_activation_scale(dev(x), 0.5)
    s_ref = O.activation_scale(x, 0.5)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))
    xs_ref = O.scale_activations(x, s_ref)
    assert np.array_equal(f16_bits(host(xs)), f16_bits(xs_ref))
    # the stored-s form gives the same bits
    xs2 = P.awq_scale_activations(dev(x), dev(s_ref))
    assert np.array_equal(f16_bits(host(xs2)), f16_bits(xs_ref))


@pytest.mark.parametrize("alpha", [0.0, 0.25, 1.0, 0.75])
def test_activation_scale_other_alpha(alpha):
    P = lib()
    x, _ = workloads.random_case(12, 64, 16, 1024)
    s, _ = P.awq_activation_scale(dev(x), alpha, want_scaled=False)
    s_ref = O.activation_scale(x, alpha)
    ulps = np.abs(host(s).view(np.int32).astype(np.int64) - s_ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1


def test_activation_scale_zero_and_constant_columns():
    P = lib()
    x = np.zeros((5, 256), np.float16)
    x[:, 1] = 3.0
    x[:, 2] = -0.5
    x[2, 3] = 65504
    s, xs = P.awq_activation_scale(dev(x), 0.5)
    s_ref = O.activation_scale(x, 0.5)
    assert np.array_equal(host(s).view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(f16_bits(host(xs)), f16_bits(O.scale_activations(x, s_ref)))


# ----------------------------------------------------------------------------- a2
def _quant_check(W, s, N, K):
    P = lib()
    packed_ref, _ = oracle_packed(W, s)
    qw, sc, zb = P.awq_quantize_g128(dev(W), dev(s) if s is not None else None)
    assert np.array_equal(host(qw).view(np.uint32), packed_ref[0]), "codes"
    assert np.array_equal(f16_bits(host(sc)), f16_bits(packed_ref[1])), "scales"
    assert np.array_equal(host(zb), packed_ref[2]), "zeros"


@pytest.mark.parametrize("N,K,fold", [(128, 128, False), (200, 384, False), (512, 512, True), (1000, 1280, True),
                                      (16, 256, True), (4096, 4096, True), (300, 11008, True)])
def test_quantize_bit_exact(N, K, fold):
    x, W = workloads.random_case(21, 4, N, K)
    s = O.activation_scale(x) if fold else None
    _quant_check(W, s, N, K)


def test_quantize_tiny_workload_with_awq_fold():
    wl = workloads.WORKLOADS["tiny_512"]
    x, W = workloads.layer_inputs(wl, 0, 1)
    _quant_check(W, O.activation_scale(x), 512, 512)


def test_quantize_hand_groups_and_extremes():
    import json, os
    fx = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "quantizer_hand_cases.json")))
    rows = []
    for c in fx["groups"]:
        rows.append(list(c["values"]) + [c["fill"]] * (128 - len(c["values"])))
    rng = np.random.default_rng(3)
    rows.append(list(np.where(rng.random(128) < 0.5, 65504.0, -65504.0)))     # full fp16 range
    rows.append([6e-8 * (i % 3) for i in range(128)])                          # subnormals
    rows.append([float(v) for v in rng.standard_normal(128) * 1e-3])
    W = np.array(rows * 3, dtype=np.float16)[:, :]                               # 36 rows
    W = np.concatenate([W, W[:, ::-1]], axis=1)                                # K = 256
    _quant_check(W, None, W.shape[0], W.shape[1])
    # with a fold scale, including values that overflow fp16 after the fold
    s = np.ones(256, np.float32)
    s[:8] = 4096.0
    s[8:16] = 1e-3
    _quant_check(W, s, W.shape[0], 256)


def _exhaustive_groups(lo, hi):
    """Rows of 128-weight groups: each group holds lo and hi (which fix S and z) and 126 fp16 values
    from [lo, hi]; together the groups hold every finite fp16 value in that interval."""
    allv = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    allv = allv[np.isfinite(allv)]
    vals = allv[(allv >= np.float16(lo)) & (allv <= np.float16(hi))]
    vals = np.unique(vals.astype(np.float32)).astype(np.float16)          # -0 and +0 once
    n = -(-len(vals) // 126)
    body = np.resize(vals, n * 126).reshape(n, 126)                        # wraps around to fill
    g = np.empty((n, 128), np.float16)
    g[:, 0], g[:, 1], g[:, 2:] = np.float16(lo), np.float16(hi), body
    return g


@pytest.mark.parametrize("fold", [False, True])
def test_quantize_every_fp16_value_over_scale_ranges(fold):
    """Every finite fp16 value is coded in groups whose bounds fix S across the whole range of
    scales: the 1e-5 floor (0x000b), subnormal S, S around 1, large S and the full fp16 range.
    This drives the exact three-operation division and both clamp paths with every operand."""
    bounds = [(0.0, 0.0), (-1e-6, 1e-6), (-2.0 ** -14, 2.0 ** -13), (-1.0, 1.0), (-7.0, 8.0), (0.5, 3.0),
              (-9.0, -2.0), (-1000.0, 250.0), (-65504.0, 65504.0)]
    groups = np.concatenate([_exhaustive_groups(lo, hi) for lo, hi in bounds])
    # rows of K = 2048 (16 groups); pad the last row with copies of the first group
    per_row = 16
    nrows = -(-len(groups) // per_row)
    groups = np.concatenate([groups, np.repeat(groups[:1], nrows * per_row - len(groups), axis=0)])
    W = groups.reshape(nrows, per_row * 128)
    s = np.ones(W.shape[1], np.float32) if fold else None
    _quant_check(W, s, W.shape[0], W.shape[1])


def _full_layer_quant_check(W, s, rows_per_chunk=2048):
    """Quantize a whole layer on the GPU; compare every packed byte with the oracle's codes packed by
    the oracle's packer, chunk by chunk of rows (a tile's codes, scales and zeros are contiguous)."""
    P = lib()
    N, K = W.shape
    qw, sc, zb = P.awq_quantize_g128(dev(W), dev(s) if s is not None else None)
    qw, sc, zb = host(qw).view(np.uint32), f16_bits(host(sc)), host(zb)
    _, _, G2, KTp = O.layout_dims(N, K)
    for r0 in range(0, N, rows_per_chunk):
        r1 = min(N, r0 + rows_per_chunk)
        t0, t1 = r0 // 16, -(-r1 // 16)
        q_ref, S_ref, z_ref = O.pack(*O.quantize_groups(O.fold_weights(W[r0:r1], s)))
        assert np.array_equal(qw[t0 * KTp * 128:t1 * KTp * 128], q_ref), f"codes, rows {r0}..{r1}"
        assert np.array_equal(sc[t0 * 2 * G2 * 16:t1 * 2 * G2 * 16], f16_bits(S_ref)), f"scales, rows {r0}..{r1}"
        assert np.array_equal(zb[t0 * 2 * G2 * 8:t1 * 2 * G2 * 8], z_ref), f"zeros, rows {r0}..{r1}"


@pytest.mark.parametrize("wl_name,li", [("llama2_70b_layers", 0), ("llama2_70b_layers", 1),
                                        ("llama2_7b_decode_m1", 0), ("llama2_7b_decode_m1", 1),
                                        ("llama2_7b_decode_m1", 2), ("llama2_7b_decode_m1", 3),
                                        ("llama3_8b_prefill", 0), ("llama3_8b_prefill", 2),
                                        ("llama3_8b_prefill", 3)])
def test_quantize_full_layer_bit_exact(wl_name, li):
    """Every packed byte of a full-size layer (with the AWQ fold from that layer's activations)."""
    wl = workloads.WORKLOADS[wl_name]
    x, W = workloads.layer_inputs(wl, li, wl.Ms[0])
    _full_layer_quant_check(W, O.activation_scale(x))


# ----------------------------------------------------------------------------- a3 / a4
LIN_SHAPES = [(512, 512), (200, 384), (1000, 1280), (4096, 4096), (136, 2304)]


def _pipeline(x, W, fn, alpha=0.5):
    """Whole path on the GPU: a1 -> a2 -> linear."""
    P = lib()
    N = W.shape[0]
    s, xs = P.awq_activation_scale(dev(x), alpha)
    qw, sc, zb = P.awq_quantize_g128(dev(W), s)
    return host(getattr(P, fn)(xs, qw, sc, zb, N)).astype(np.float64)


@pytest.mark.parametrize("N,K", LIN_SHAPES)
@pytest.mark.parametrize("M", [1, 2, 5, 8, 9, 16, 23, 32])
def test_gemv_whole_path(M, N, K):
    x, W = workloads.random_case(31 + M, M, N, K)
    r = O.reference_forward(x, W)
    y = _pipeline(x, W, "awq_w4a16_gemv")
    assert_tolerance(y, r["y"], f"gemv M={M} N={N} K={K}")
    assert_tight(y, r["y"], what="gemv")


@pytest.mark.parametrize("M", [1, 3, 8, 17, 32])
def test_gemv_on_oracle_packed_weights(M):
    """The decode kernel alone, fed the oracle's packed weights and the oracle's x'."""
    P = lib()
    N, K = 1000, 2304
    x, W = workloads.random_case(41, M, N, K)
    r = O.reference_forward(x, W)
    qw, sc, zb = upload_packed(O.pack(r["q"], r["S"], r["z"]))
    y = host(P.awq_w4a16_gemv(dev(r["xs"]), qw, sc, zb, N)).astype(np.float64)
    assert_tolerance(y, r["y"], "gemv isolated")
    assert_tight(y, r["y"], what="gemv isolated")


@pytest.mark.parametrize("N,K", LIN_SHAPES)
@pytest.mark.parametrize("M", [1, 17, 33, 64, 100, 128, 129, 256, 300, 513])
def test_gemm_whole_path(M, N, K):
    x, W = workloads.random_case(51 + M, M, N, K)
    r = O.reference_forward(x, W)
    y = _pipeline(x, W, "awq_w4a16_gemm")
    assert_tolerance(y, r["y"], f"gemm M={M} N={N} K={K}")
    assert_tight(y, r["y"], rel=2.0 ** -10, abs_rms=3e-3, what="gemm")


@pytest.mark.parametrize("M", [40, 200, 1024])
def test_gemm_on_oracle_packed_weights(M):
    P = lib()
    N, K = 1000, 2304
    x, W = workloads.random_case(61, M, N, K)
    r = O.reference_forward(x, W)
    qw, sc, zb = upload_packed(O.pack(r["q"], r["S"], r["z"]))
    y = host(P.awq_w4a16_gemm(dev(r["xs"]), qw, sc, zb, N)).astype(np.float64)
    assert_tolerance(y, r["y"], "gemm isolated")
    assert_tight(y, r["y"], rel=2.0 ** -10, abs_rms=3e-3, what="gemm isolated")


def test_linear_dispatch_and_determinism():
    P = lib()
    for M in (4, 32, 33, 200):
        x, W = workloads.random_case(71, M, 512, 1024)
        s, xs = P.awq_activation_scale(dev(x))
        qw, sc, zb = P.awq_quantize_g128(dev(W), s)
        y1 = host(P.awq_w4a16_linear(xs, qw, sc, zb, 512))
        ref = P.awq_w4a16_gemv if M <= 32 else P.awq_w4a16_gemm
        y2 = host(ref(xs, qw, sc, zb, 512))
        y3 = host(ref(xs, qw, sc, zb, 512))
        assert np.array_equal(f16_bits(y1), f16_bits(y2)) and np.array_equal(f16_bits(y2), f16_bits(y3))


# ----------------------------------------------------------------------------- full sizes, sampled outputs
def _sampled_reference(x, W, rows, toks):
    """y_ref[toks][:, rows] computed by the oracle from the seeded x, W only."""
    s = O.activation_scale(x)
    xs = O.scale_activations(x[toks], s)
    q, S, z = O.quantize_groups(O.fold_weights(W[rows], s))
    return O.linear(xs, O.dequantize(q, S, z))


def _full_size_case(wl_name, layer_idx, M, fn, n_rows=192, n_toks=24):
    wl = workloads.WORKLOADS[wl_name]
    x, W = workloads.layer_inputs(wl, layer_idx, M)
    N = W.shape[0]
    y = _pipeline(x, W, fn)
    rng = np.random.default_rng(layer_idx * 1000 + M)
    rows = np.unique(np.concatenate([[0, N - 1], rng.choice(N, n_rows, replace=False)]))
    toks = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(M, n_toks), replace=False)]))
    y_ref = _sampled_reference(x, W, rows, toks)
    got = y[np.ix_(toks, rows)]
    assert_tolerance(got, y_ref, f"{wl_name}[{layer_idx}] M={M}")
    assert_tight(got, y_ref, rel=2.0 ** -10, abs_rms=3e-3, what=f"{wl_name}[{layer_idx}] M={M}")


@pytest.mark.parametrize("layer_idx", [0, 1, 2, 3])
def test_decode_m1_full_size_sampled(layer_idx):
    _full_size_case("llama2_7b_decode_m1", layer_idx, 1, "awq_w4a16_gemv")


@pytest.mark.parametrize("M", [4, 8, 16, 32])
@pytest.mark.parametrize("layer_idx", [0, 1, 2, 3])
def test_batched_decode_full_size_sampled(layer_idx, M):
    """Every (layer, M) pair of the Llama-2-7B batched decode set, through the dispatching call."""
    _full_size_case("llama2_7b_decode_batched", layer_idx, M, "awq_w4a16_linear")


@pytest.mark.parametrize("M", [512, 2048, 4096])
@pytest.mark.parametrize("layer_idx", [0, 1, 2, 3])
def test_prefill_full_size_sampled(layer_idx, M):
    """Every (layer, M) pair of the Llama-3-8B prefill set."""
    _full_size_case("llama3_8b_prefill", layer_idx, M, "awq_w4a16_gemm")


@pytest.mark.parametrize("M", [1, 16, 512])
@pytest.mark.parametrize("layer_idx", [0, 1])
def test_70b_full_size_sampled(layer_idx, M):
    """Every (layer, M) pair of the Llama-2-70B set, through the dispatching call."""
    _full_size_case("llama2_70b_layers", layer_idx, M, "awq_w4a16_linear")


@pytest.mark.parametrize("M", [1, 2, 9, 64])
@pytest.mark.parametrize("N", [16, 200])
def test_single_group_k128(M, N):
    """K = 128: one group per row (G = 1, so one padding group per tile), both kernels."""
    x, W = workloads.random_case(61 + M, M, N, 128)
    r = O.reference_forward(x, W)
    for fn in (["awq_w4a16_gemv"] if M <= 32 else []) + ["awq_w4a16_gemm"]:
        y = _pipeline(x, W, fn)
        assert_tolerance(y, r["y"], f"{fn} K=128 M={M} N={N}")
        assert_tight(y, r["y"], what=f"{fn} K=128")


# ----------------------------------------------------------------------------- launch chaining
@pytest.mark.parametrize("use_graph", [False, True])
def test_decode_chained_on_requantized_buffers(use_graph):
    """a1 -> a2 -> a3 for three different layers into the SAME packed buffers, launched back to back
    on one stream with no host synchronization (eagerly, and captured in a CUDA graph, which keeps
    programmatic dependent launch). Each decode reads weights that the immediately preceding
    quantizer wrote, and each quantizer overwrites weights the previous decode read: the decode
    kernel's early weight reads must still see complete, current weights."""
    P = lib()
    torch = torch_mod()
    N, K = 2048, 4096
    cases = [workloads.random_case(121 + i, 1 + i, N, K) for i in range(3)]
    dx = [dev(x) for x, _ in cases]
    dW = [dev(W) for _, W in cases]
    packed = P.alloc_packed(N, K)
    s = [torch.empty(K, dtype=torch.float32, device="cuda") for _ in cases]
    xs = [torch.empty_like(x) for x in dx]
    ys = [torch.empty((x.shape[0], N), dtype=torch.float16, device="cuda") for x in dx]

    def chain():
        for i in range(len(cases)):
            P.awq_activation_scale(dx[i], 0.5, s[i], xs[i])
            P.awq_quantize_g128(dW[i], s[i], packed)
            P.awq_w4a16_gemv(xs[i], *packed, N, ys[i])

    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        chain()   # eager run (also sets kernel attributes before any capture)
        if use_graph:
            for y in ys:
                y.zero_()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                chain()
            g.replay()
        stream.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK
    for i, (x, W) in enumerate(cases):
        r = O.reference_forward(x, W)
        if i == len(cases) - 1:   # the buffers hold the last layer's codes
            assert np.array_equal(host(packed[0]).view(np.uint32), O.pack(r["q"], r["S"], r["z"])[0])
        y = host(ys[i]).astype(np.float64)
        assert_tolerance(y, r["y"], f"chained layer {i}")
        assert_tight(y, r["y"], what=f"chained layer {i}")
