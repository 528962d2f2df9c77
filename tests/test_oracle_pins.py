"""Pins for the CPU oracle, against things other than the oracle itself.

Each test ties one oracle function to something fixed outside it: hand-derived
golden fixtures (``tests/golden/``), brute-force search, closed forms, exact
rational arithmetic, or invariants the method guarantees. A plausible slip in
the oracle (a swapped min/max, a floor for a rint, a transposed operand, a
fold applied the wrong way round, a wrong index in the layout) fails one of
them. None of these tests needs a GPU.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f16_bits(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


# ----------------------------------------------------------------------------
# quantizer: hand-derived groups
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("case", _load("quantizer_hand_cases.json")["groups"], ids=lambda c: c["name"])
def test_quantizer_hand_cases(case):
    vals = list(case["values"]) + [case["fill"]] * (128 - len(case["values"]))
    W = np.array([vals], dtype=np.float16)
    assert np.all(W.astype(np.float64) == np.array([vals])), "fixture values must be fp16-exact"
    q, S, z = O.quantize_groups(W)
    expect = list(case["codes"]) + [case["fill_code"]] * (128 - len(case["codes"]))
    assert q[0].tolist() == expect
    assert int(_f16_bits(S)[0, 0]) == int(case["scale_bits"], 16)
    assert int(z[0, 0]) == case["zero"]


def test_quantizer_groups_are_independent_and_rows_too():
    """Two hand groups side by side in one row, and stacked rows, give the same results."""
    cases = _load("quantizer_hand_cases.json")["groups"]
    rows = []
    for c in cases:
        rows.append(list(c["values"]) + [c["fill"]] * (128 - len(c["values"])))
    a = np.array(rows, dtype=np.float16)
    wide = np.concatenate([a, a[::-1]], axis=1)            # [n, 256]: 2 groups per row
    q, S, z = O.quantize_groups(wide)
    q1, S1, z1 = O.quantize_groups(a)
    q2, S2, z2 = O.quantize_groups(a[::-1])
    assert np.array_equal(q[:, :128], q1) and np.array_equal(q[:, 128:], q2)
    assert np.array_equal(_f16_bits(S[:, 0]), _f16_bits(S1[:, 0]))
    assert np.array_equal(_f16_bits(S[:, 1]), _f16_bits(S2[:, 0]))
    assert np.array_equal(z[:, 0], z1[:, 0]) and np.array_equal(z[:, 1], z2[:, 0])


# ----------------------------------------------------------------------------
# quantizer: brute-force nearest level
# ----------------------------------------------------------------------------
def _brute_codes(w32, S16):
    """q = the level c in 0..15 whose value (c - z) is nearest to w/S (fp32 quotient).

    z itself is the integer in 0..15 nearest to -lo/S. Ties go to the even
    integer (of c - z, resp. of z), which is what round-half-even means.
    """
    Sf = np.float32(S16)
    lo = np.float32(np.min(w32))
    t = float(np.float32(-lo) / Sf)
    best = None
    for c in range(16):
        d = abs(t - c)
        key = (d, c % 2)
        if best is None or key < best[0]:
            best = (key, c)
    zb = best[1]
    out = []
    for w in w32:
        v = float(np.float32(w) / Sf)
        best = None
        for c in range(16):
            d = abs(v - (c - zb))
            key = (d, (c - zb) % 2)
            if best is None or key < best[0]:
                best = (key, c)
        out.append(best[1])
    return np.array(out, dtype=np.uint8), zb


def test_quantizer_brute_force_random_groups():
    rng = np.random.default_rng(1234)
    for trial in range(60):
        kind = trial % 4
        if kind == 0:
            w = rng.standard_normal(128) * 0.02
        elif kind == 1:
            w = rng.standard_normal(128) * 3.0 + rng.uniform(-2, 2)
        elif kind == 2:
            w = rng.uniform(0.5, 1.5, 128)           # all positive: z clamps at 0
        else:
            w = -rng.uniform(0.5, 1.5, 128)          # all negative: z clamps at 15
        W = w.astype(np.float16)[None, :]
        q, S, z = O.quantize_groups(W)
        qb, zb = _brute_codes(W[0].astype(np.float32), S[0, 0])
        assert int(z[0, 0]) == zb
        assert np.array_equal(q[0], qb), f"trial {trial}"


def test_quantizer_exhaustive_fp16_grid_unit_scale():
    """Every finite fp16 value in [-7, 8] placed in a group whose min/max are -7 and 8.

    Then S = 1, z = 7 and the code of w must be clamp(rint(w) + 7): brute
    force over the 16 levels decides it, ties to the even level.
    """
    bits = np.arange(0x10000, dtype=np.uint32).astype(np.uint16)
    vals = bits.view(np.float16)
    vals = vals[np.isfinite(vals)]
    vals = vals[(vals >= -7) & (vals <= 8)]
    vals = np.unique(vals.astype(np.float32))        # one -0/0 only
    n = len(vals)
    per = 126
    rows = -(-n // per)
    W = np.zeros((rows, 128), dtype=np.float16)
    W[:, 0] = -7
    W[:, 1] = 8
    flat = np.zeros(rows * per, dtype=np.float32)
    flat[:n] = vals
    W[:, 2:] = flat.reshape(rows, per).astype(np.float16)
    q, S, z = O.quantize_groups(W)
    assert np.all(S.astype(np.float32) == 1.0) and np.all(z == 7)
    got = q[:, 2:].reshape(-1)[:n]
    # brute force with S = 1, z = 7 (v = w exactly)
    levels = np.arange(16, dtype=np.float64) - 7
    d = np.abs(vals.astype(np.float64)[:, None] - levels[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = (d == dmin)
    even = (np.mod(levels, 2) == 0)[None, :]
    pick = np.where(cand & even, 1, 0) * 2 + np.where(cand, 1, 0)
    expect = np.argmax(pick, axis=1)
    assert np.array_equal(got.astype(np.int64), expect)


# ----------------------------------------------------------------------------
# quantizer: invariants on the synthetic recipe
# ----------------------------------------------------------------------------
def test_quantizer_invariants_on_recipe():
    x, W = workloads.random_case(7, 4, 256, 1024)
    s = O.activation_scale(x)
    wf = O.fold_weights(W, s)
    q, S, z = O.quantize_groups(wf)
    assert q.dtype == np.uint8 and q.max() <= 15 and z.max() <= 15
    N, K = wf.shape
    G = K // 128
    wg = wf.astype(np.float64).reshape(N, G, 128)
    Sd = S.astype(np.float64)
    lo, hi = wg.min(axis=2), wg.max(axis=2)
    # the scale is (hi - lo)/15 up to one fp32 and one fp16 rounding
    ratio = (hi - lo) / Sd / 15.0
    assert np.all(np.abs(ratio - 1) <= 2.0 ** -11 + 2.0 ** -23)
    # the group minimum lands on code 0 when z is not clamped
    qg = q.reshape(N, G, 128)
    argmin = wg.argmin(axis=2)
    qlo = np.take_along_axis(qg, argmin[..., None], axis=2)[..., 0]
    unclamped = (-lo / Sd) <= 15.5
    assert np.all(qlo[unclamped] == 0)
    # dequantization error <= S/2, except codes clamped at 15 (rounded S), by at most 15 * 2^-11 S
    what = O.dequantize(q, S, z).reshape(N, G, 128)
    err = np.abs(what - wg)
    assert np.all(err <= Sd[..., None] * (0.5 + 0.008))
    over = err > Sd[..., None] * 0.5 * (1 + 1e-12)
    assert np.all(qg[over] == 15)


# ----------------------------------------------------------------------------
# dequantization and matmul: exact rational arithmetic
# ----------------------------------------------------------------------------
def test_dequantize_exact_rational():
    rng = np.random.default_rng(5)
    q = rng.integers(0, 16, (3, 256)).astype(np.uint8)
    z = rng.integers(0, 16, (3, 2)).astype(np.uint8)
    S = (rng.uniform(1e-4, 2.0, (3, 2))).astype(np.float16)
    d = O.dequantize(q, S, z)
    for n in range(3):
        for k in range(0, 256, 7):
            g = k // 128
            exact = (Fraction(int(q[n, k])) - int(z[n, g])) * Fraction(float(S[n, g]))
            assert Fraction(float(d[n, k])) == exact


def test_linear_matches_exact_rationals():
    rng = np.random.default_rng(11)
    for (M, K, N) in [(1, 128, 3), (4, 256, 16), (2, 128, 5)]:
        xs = rng.standard_normal((M, K)).astype(np.float16)
        w = rng.standard_normal((N, K)).astype(np.float16).astype(np.float64)
        y = O.linear(xs, w)
        assert y.shape == (M, N)
        for m in range(M):
            for n in range(N):
                ex = sum(Fraction(float(xs[m, k])) * Fraction(float(w[n, k])) for k in range(K))
                assert abs(float(ex) - y[m, n]) <= 1e-12 * max(1.0, abs(float(ex)))


# ----------------------------------------------------------------------------
# activation statistic, activation scaling, fold
# ----------------------------------------------------------------------------
def test_activation_scale_closed_forms():
    x = np.array([[0, 1, 4, -9, 0.5],
                  [0, -1, 0, -16, 0.5]], dtype=np.float16)
    s = O.activation_scale(x)
    expect = [math.sqrt(1e-8), 1.0, math.sqrt(2.0), math.sqrt(12.5), math.sqrt(0.5)]
    assert s.dtype == np.float32
    assert s.tolist() == [float(np.float32(e)) for e in expect]
    # alpha = 1 gives the mean, alpha = 0 gives 1
    s1 = O.activation_scale(x, alpha=1.0)
    assert s1.tolist() == [float(np.float32(e)) for e in [1e-8, 1.0, 2.0, 12.5, 0.5]]
    assert np.all(O.activation_scale(x, alpha=0.0) == 1.0)


def test_activation_scale_exact_mean():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((37, 64)) * 30).astype(np.float16)
    s = O.activation_scale(x, alpha=1.0)
    for j in range(64):
        mean = sum(Fraction(abs(float(v))) for v in x[:, j]) / 37
        assert float(s[j]) == float(np.float32(float(mean)))


def test_scale_activations_closed_form():
    x = np.array([[1.0, -3.0, 0.0]], dtype=np.float16)
    s = np.array([math.sqrt(2.0), 0.5, 7.0], dtype=np.float32)
    xs = O.scale_activations(x, s)
    # 1/1.4142135 = 0.70710677 -> fp16 0.70703125 (0x39a8); -3/0.5 = -6; 0/7 = 0
    assert _f16_bits(xs)[0].tolist() == [0x39A8, int(_f16_bits(np.float16(-6.0))), 0]


def test_fold_direction_equivalence_exact():
    """(W diag(s)) (diag(1/s) x) = W x, computed exactly, so the fold goes on columns k."""
    rng = np.random.default_rng(9)
    M, N, K = 3, 5, 256
    x, W = workloads.random_case(9, M, N, K)
    s = O.activation_scale(x)
    # exact float64 version of both halves of the transform
    Wd = W.astype(np.float64) * s.astype(np.float64)[None, :]
    xd = x.astype(np.float64) / s.astype(np.float64)[None, :]
    lhs = xd @ Wd.T
    rhs = x.astype(np.float64) @ W.astype(np.float64).T
    assert np.allclose(lhs, rhs, rtol=1e-12, atol=1e-12 * np.abs(rhs).max())
    # the stored (fp16-rounded) halves keep the product to fp16 accuracy
    y16 = O.scale_activations(x, s).astype(np.float64) @ O.fold_weights(W, s).astype(np.float64).T
    assert np.linalg.norm(y16 - rhs) / np.linalg.norm(rhs) < 2e-3
    # the weight side is the one scaled UP on large-activation channels, column by column
    wf = O.fold_weights(W, s).astype(np.float64)
    j = int(np.argmax(s))
    assert s[j] > 2
    ratio = wf[:, j] / W[:, j].astype(np.float64)
    assert np.allclose(ratio, s[j], rtol=2e-3)
    xs = O.scale_activations(x, s).astype(np.float64)
    assert np.allclose(xs[:, j] * s[j], x[:, j].astype(np.float64), rtol=2e-3)


def test_awq_scaling_reduces_error_on_outlier_recipe():
    """The method's claim: scaling salient (large-activation) channels lowers the output error."""
    wl = workloads.WORKLOADS["tiny_512"]
    x, W = workloads.layer_inputs(wl, 0, 1)
    exact = x.astype(np.float64) @ W.astype(np.float64).T
    r = O.reference_forward(x, W)
    plain = O.linear(x, O.fake_quantize(W, None))
    e_awq = np.linalg.norm(r["y"] - exact) / np.linalg.norm(exact)
    e_rtn = np.linalg.norm(plain - exact) / np.linalg.norm(exact)
    assert e_awq < e_rtn
    assert e_awq < 0.1


def test_fold_none_is_identity():
    _, W = workloads.random_case(2, 1, 7, 128)
    assert np.array_equal(O.fold_weights(W, None).view(np.uint16), W.view(np.uint16))


# ----------------------------------------------------------------------------
# packed layout
# ----------------------------------------------------------------------------
def test_layout_hand_positions():
    fx = _load("layout_positions.json")
    for shp in fx["shapes"]:
        N, K = shp["N"], shp["K"]
        G = K // 128
        words, nsc, nzb = O.packed_sizes(N, K)
        assert (words, nsc, nzb) == (shp["sizes"]["words"], shp["sizes"]["scales"], shp["sizes"]["zero_bytes"])
        for c in shp["codes"]:
            q = np.zeros((N, K), np.uint8)
            q[c["n"], c["k"]] = 0xB
            qw, _, _ = O.pack(q, np.zeros((N, G), np.float16), np.zeros((N, G), np.uint8))
            nz = np.nonzero(qw)[0]
            assert nz.tolist() == [c["word"]]
            assert int(qw[c["word"]]) == 0xB << (4 * c["nibble"])
        for c in shp["scales"]:
            S = np.zeros((N, G), np.float16)
            S[c["n"], c["g"]] = 1.0
            _, sc, _ = O.pack(np.zeros((N, K), np.uint8), S, np.zeros((N, G), np.uint8))
            assert np.nonzero(sc)[0].tolist() == [c["index"]]
        for c in shp["zeros"]:
            z = np.zeros((N, G), np.uint8)
            z[c["n"], c["g"]] = 9
            _, _, zb = O.pack(np.zeros((N, K), np.uint8), np.zeros((N, G), np.float16), z)
            assert np.nonzero(zb)[0].tolist() == [c["byte"]]
            assert int(zb[c["byte"]]) == (9 << 4 if c["high"] else 9)


@pytest.mark.parametrize("N,K", [(128, 128), (300, 256), (16, 384), (513, 640), (7, 1152)])
def test_layout_roundtrip(N, K):
    rng = np.random.default_rng(N * 31 + K)
    G = K // 128
    q = rng.integers(0, 16, (N, K)).astype(np.uint8)
    S = rng.standard_normal((N, G)).astype(np.float16)
    z = rng.integers(0, 16, (N, G)).astype(np.uint8)
    qw, sc, zb = O.pack(q, S, z)
    assert (qw.size, sc.size, zb.size) == O.packed_sizes(N, K)
    q2, S2, z2 = O.unpack(qw, sc, zb, N, K)
    assert np.array_equal(q, q2) and np.array_equal(S.view(np.uint16), S2.view(np.uint16))
    assert np.array_equal(z, z2)
    # padding rows and padding groups decode as zeros
    Np = O.padded_rows(N)
    NT, _, G2, KTp = O.layout_dims(N, K)
    qa, Sa, za = O.unpack(qw, sc, zb, Np, 128 * 2 * G2)
    assert not qa[N:].any() and not qa[:, K:].any()
    assert not Sa[N:].astype(np.float32).any() and not Sa[:, G:].astype(np.float32).any()
    assert not za[N:].any() and not za[:, G:].any()


def test_layout_lane_chunk_holds_its_fragment():
    """A lane's 16 bytes (4 words) hold rows r, r+8 and k in [16t, 16t+16) of one 16x64 tile, and a tile's
    64-k tiles follow one another in memory."""
    N, K = 128, 256
    G = 2
    for (T, r, t, kt) in [(0, 0, 0, 0), (3, 5, 2, 1), (7, 7, 3, 3)]:
        mark = np.zeros((N, K), np.uint8)
        rows = [T * 16 + r, T * 16 + r + 8]
        cols = slice(kt * 64 + 16 * t, kt * 64 + 16 * t + 16)
        mark[rows[0], cols] = 1
        mark[rows[1], cols] = 1
        qw, _, _ = O.pack(mark * 15, np.zeros((N, G), np.float16), np.zeros((N, G), np.uint8))
        lane = 4 * r + t
        base = (T * 4 + kt) * 128 + lane * 4
        assert np.nonzero(qw)[0].tolist() == [base, base + 1, base + 2, base + 3]
        assert all(int(w) == 0xFFFFFFFF for w in qw[base:base + 4])


def test_layout_tile_streams_are_contiguous():
    """Everything of tile T (codes, scales, zeros) lies in one contiguous range of each array, in k order."""
    N, K = 64, 512
    NT, G, G2, KTp = O.layout_dims(N, K)
    for T in range(NT):
        q = np.zeros((N, K), np.uint8)
        q[16 * T:16 * T + 16] = 15
        S = np.zeros((N, G), np.float16)
        S[16 * T:16 * T + 16] = 1.0
        z = np.zeros((N, G), np.uint8)
        z[16 * T:16 * T + 16] = 15
        qw, sc, zb = O.pack(q, S, z)
        assert np.nonzero(qw)[0].tolist() == list(range(T * KTp * 128, (T + 1) * KTp * 128))
        assert np.nonzero(sc)[0].tolist() == list(range(T * 2 * G2 * 16, (T + 1) * 2 * G2 * 16))
        assert np.nonzero(zb)[0].tolist() == list(range(T * 2 * G2 * 8, (T + 1) * 2 * G2 * 8))


# ----------------------------------------------------------------------------
# tolerance check helper and the configuration contract
# ----------------------------------------------------------------------------
def test_check_tolerance_boundaries():
    rng = np.random.default_rng(0)
    y = rng.standard_normal((4, 64))
    ok, ef, em = O.check_tolerance(y, y)
    assert ok and ef == 0 and em == 0
    rms = np.sqrt(np.mean(y ** 2))
    bump = y.copy()
    bump[0, 0] += 0.011 * rms          # max error just above 1e-2 rms
    assert not O.check_tolerance(bump, y)[0]
    bump[0, 0] = y[0, 0] + 0.009 * rms
    assert O.check_tolerance(bump, y)[0]
    assert not O.check_tolerance(y * (1 + 3e-3), y)[0]    # Frobenius 3e-3


def test_quant_config_fixture_is_the_built_configuration():
    fx = _load("quant_configs.json")
    hf = fx["hf_quantization_config"]
    assert (hf["bits"], hf["group_size"], hf["zero_point"]) == (O.BITS, O.GROUP_SIZE, True)
    aw = fx["autoawq_quant_config"]
    assert (aw["w_bit"], aw["q_group_size"], aw["zero_point"]) == (O.BITS, O.GROUP_SIZE, True)
    assert O.QMAX == 2 ** O.BITS - 1


def test_reference_forward_tiny_workload_shapes():
    wl = workloads.WORKLOADS["tiny_512"]
    x, W = workloads.layer_inputs(wl, 0, 1)
    r = O.reference_forward(x, W)
    assert r["q"].shape == (512, 512) and r["S"].shape == (512, 4) and r["y"].shape == (1, 512)
    assert workloads.n_outlier_channels(512) == 5


# ----------------------------------------------------------------------------
# AWQ scale search
# ----------------------------------------------------------------------------
def _search_case_known_optimum(seed=5, M=8, N=32, K=256):
    """Calibration rows and weights for which alpha = 0.5 quantizes losslessly by construction.

    Channel j has mean |x_j| = 4^k_j (rows are +-4^k_j), so at alpha = 0.5 the scale is s_j = 2^k_j
    exactly and x' = x / s is exact. The weights are W_nj = m_nj 2^(-6 - k_j) with integer
    m_nj in 0..15 and every group holding a 0 and a 15, so W s = m 2^-6 sits exactly on the 4-bit grid
    (lo = 0, S = 2^-6, z = 0) and dequantizes to itself: the output error is exactly zero. Other
    exponents give non-power-of-two scales, off-grid folded weights and a positive error.
    """
    rng = np.random.default_rng(seed)
    k = np.array([-1, 0, 1, 2] * (K // 4))
    x = (np.where(rng.random((M, K)) < 0.5, -1.0, 1.0) * (4.0 ** k)[None, :]).astype(np.float16)
    m = rng.integers(0, 16, (N, K))
    m[:, 0::128] = 0
    m[:, 1::128] = 15
    W = (m * 2.0 ** (-6 - k)[None, :]).astype(np.float16)
    assert np.array_equal(W.astype(np.float64), m * 2.0 ** (-6 - k)[None, :])   # exact in fp16
    return x, W


def test_search_finds_the_constructed_optimum():
    x, W = _search_case_known_optimum()
    alpha, s, errs = O.search_alpha(x, W)
    assert alpha == 0.5
    assert np.array_equal(s, (2.0 ** np.array([-1, 0, 1, 2] * 64)).astype(np.float32))
    assert errs[10] == 0.0
    assert (np.delete(errs, 10) > 0).all()


def test_search_errors_definition_pieces():
    """The error at alpha = 0 is the plain quantization error of W (no fold: s = mean|x|^0 = 1 and
    x' = x), written here from the pieces, not from search_errors."""
    x, W = workloads.random_case(7, 4, 24, 256)
    errs = O.search_errors(x, W, np.array([0.0], np.float32))
    q, S, z = O.quantize_groups(W)
    w_hat = (q.astype(np.float64).reshape(24, 2, 128) - z[..., None]) * S.astype(np.float64)[..., None]
    y_q = x.astype(np.float64) @ w_hat.reshape(24, 256).T
    y = x.astype(np.float64) @ W.astype(np.float64).T
    assert abs(errs[0] - np.sum((y - y_q) ** 2)) <= 1e-12 * np.sum(y ** 2)


def test_alpha_grid_is_even_over_unit_interval():
    g = O.alpha_grid(20)
    assert g.dtype == np.float32 and g[0] == 0.0 and g[10] == 0.5 and len(g) == 20 and g[-1] < 1.0
    assert np.allclose(np.diff(g.astype(np.float64)), 0.05)


# ----------------------------------------------------------------------------
# fused epilogues
# ----------------------------------------------------------------------------
def test_silu_closed_forms():
    assert O.silu(np.array([0.0]))[0] == 0.0
    # SiLU(v) -> v for large v, -> 0 for very negative v; SiLU(ln 3) = ln(3) * 3/4
    assert abs(O.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(O.silu(np.array([-40.0]))[0]) < 1e-15
    assert abs(O.silu(np.array([np.log(3.0)]))[0] - 0.75 * np.log(3.0)) < 1e-15
    # odd part: SiLU(v) - SiLU(-v) = v
    v = np.linspace(-5, 5, 11)
    assert np.allclose(O.silu(v) - O.silu(-v), v, rtol=0, atol=1e-14)


def test_gate_up_silu_pairs_row_i_with_row_i_plus_I():
    y = np.zeros((2, 6))
    y[:, :3] = [[0.0, np.log(3.0), 1.0], [2.0, -1.0, 0.5]]
    y[:, 3:] = [[5.0, 4.0, 0.0], [1.0, 2.0, -2.0]]
    h = O.gate_up_silu(y)
    assert h.shape == (2, 3)
    assert h[0, 0] == 0.0 and abs(h[0, 1] - 3.0 * np.log(3.0)) < 1e-14 and h[0, 2] == 0.0
    assert abs(h[1, 0] - 2.0 / (1.0 + np.exp(-2.0))) < 1e-15


def test_split_qkv_blocks():
    y = np.arange(2 * 12).reshape(2, 12)
    q, k, v = O.split_qkv(y, 8, 2)
    assert q.tolist() == y[:, :8].tolist() and k.tolist() == y[:, 8:10].tolist() and v.tolist() == y[:, 10:].tolist()


# ----------------------------------------------------------------------------
# quantizer variants (INT3, symmetric, group 64)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("case", _load("quantizer_variant_cases.json")["groups"], ids=lambda c: c["name"])
def test_quantizer_variant_hand_cases(case):
    vals = list(case["values"]) + [case["fill"]] * (128 - len(case["values"]))
    W = np.array([vals], dtype=np.float16)
    assert np.all(W.astype(np.float64) == np.array([vals])), "fixture values must be fp16-exact"
    q, S, z = O.quantize_groups_cfg(W, case["bits"], 128, case["zero_point"])
    expect = list(case["codes"]) + [case["fill_code"]] * (128 - len(case["codes"]))
    assert q[0].tolist() == expect
    assert int(_f16_bits(S)[0, 0]) == int(case["scale_bits"], 16)
    assert int(z[0, 0]) == case["zero"]


def test_quantizer_cfg_default_is_the_pinned_int4_quantizer():
    W = workloads.make_weight(0, 7, 1, 48, 512)
    a = O.quantize_groups(W)
    b = O.quantize_groups_cfg(W, 4, 128, True)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))


def _brute_codes_cfg(w32, S16, qmax, z_fixed=None):
    """Nearest level c in 0..qmax of (c - z) to w/S, ties to the even integer; z as in _brute_codes
    (nearest integer in 0..qmax to -lo/S) unless fixed."""
    Sf = np.float32(S16)
    if z_fixed is None:
        t = float(np.float32(-np.float32(np.min(w32))) / Sf)
        zb = min(range(qmax + 1), key=lambda c: (abs(t - c), c % 2))
    else:
        zb = z_fixed
    out = []
    for w in w32:
        v = float(np.float32(w) / Sf)
        out.append(min(range(qmax + 1), key=lambda c: (abs(v - (c - zb)), (c - zb) % 2)))
    return np.array(out, dtype=np.uint8), zb


@pytest.mark.parametrize("bits,zero_point", [(3, True), (3, False), (4, False)])
def test_quantizer_variant_brute_force(bits, zero_point):
    rng = np.random.default_rng(77 + bits + 10 * zero_point)
    qmax = (1 << bits) - 1
    for trial in range(40):
        kind = trial % 4
        if kind == 0:
            w = rng.standard_normal(128) * 0.02
        elif kind == 1:
            w = rng.standard_normal(128) * 3.0 + rng.uniform(-2, 2)
        elif kind == 2:
            w = rng.uniform(0.5, 1.5, 128)
        else:
            w = -rng.uniform(0.5, 1.5, 128)
        W = w.astype(np.float16)[None, :]
        q, S, z = O.quantize_groups_cfg(W, bits, 128, zero_point)
        w32 = W[0].astype(np.float32)
        if not zero_point:
            # the scale itself: fp16 of max|w| / (2^(bits-1) - 1)
            a = float(np.max(np.abs(w32)))
            assert S[0, 0] == np.float16(np.float32(a) / np.float32((1 << (bits - 1)) - 1))
        qb, zb = _brute_codes_cfg(w32, S[0, 0], qmax, None if zero_point else 1 << (bits - 1))
        assert int(z[0, 0]) == zb
        assert np.array_equal(q[0], qb), f"trial {trial}"


def test_quantizer_symmetric_invariants():
    """Symmetric codes never clamp for finite groups: |w - (q - z) S| <= S/2 and q >= 1."""
    W = workloads.make_weight(3, 7, 2, 64, 1024)
    for bits in (3, 4):
        q, S, z = O.quantize_groups_cfg(W, bits, 128, False)
        assert np.all(z == (1 << (bits - 1)))
        err = np.abs(O.dequantize_cfg(q, S, z, 128) - W.astype(np.float64))
        half = np.repeat(S.astype(np.float64), 128, axis=1) / 2
        assert np.all(err <= half * (1 + 1e-6))
        assert q.min() >= 1 and q.max() <= (1 << bits) - 1


def test_quantizer_group64_equals_group128_of_duplicated_halves():
    """A 64-wide group's min, max and codes are those of a 128-wide group holding it twice."""
    W = workloads.make_weight(5, 7, 3, 16, 512)
    for bits, zp in ((4, True), (3, False)):
        q64, S64, z64 = O.quantize_groups_cfg(W, bits, 64, zp)
        halves = W.reshape(16, 8, 64)
        dup = np.concatenate([halves, halves], axis=2).reshape(16, 1024)
        q128, S128, z128 = O.quantize_groups_cfg(dup, bits, 128, zp)
        assert np.array_equal(q64.reshape(16, 8, 64), q128.reshape(16, 8, 128)[:, :, :64])
        assert np.array_equal(_f16_bits(S64), _f16_bits(S128)) and np.array_equal(z64, z128)
        # and dequantization respects the group width
        wh = O.dequantize_cfg(q64, S64, z64, 64)
        assert np.array_equal(wh, O.dequantize_cfg(q128, S128, z128, 128).reshape(16, 8, 128)[:, :, :64].reshape(16, 512))
