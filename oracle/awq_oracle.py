"""CPU oracle for the AWQ W4A16 g128 path — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this module. The CUDA library never calls it, links it or
falls back to it, and it shares no code with the CUDA path: the packed layout
below is restated here from its written specification, not imported.

Plain NumPy, written for a reader to check by eye against the pages. Every
floating-point step that decides an integer (a code, a zero point) is taken in
IEEE fp32 with round-to-nearest-even, the same precision the CUDA quantizer
uses; the matmul is float64.

Sources (page title, section):

* [AWQ-README] "AWQ: Activation-aware Weight Quantization for LLM Compression
  and Acceleration" (llm-awq README mirror on dongaigc.com): "Usage" steps
  1-3 (``--w_bit 4 --q_group_size 128``; ``--q_backend fake`` simulated
  quantization; ``--q_backend real`` packed INT4), "Installation" step 3
  (W4A16 = 4-bit weights, 16-bit activations).
* [HF-AWQ] "transformers - AWQ" (coreui.cn translation of the HF guide),
  section 2 ("quantization_config": quant_method awq, zero_point true,
  group_size 128, bits 4, version gemm).
* [AutoAWQ-blog] "AWQ (Activation-Aware Weight Quantization) and its
  differences from GPTQ" (llmstudio.ru), section "Quantizing a model with
  AutoAWQ": w_bit, q_group_size (scale and zero point shared by a group),
  zero_point = asymmetric quantization.
* [CSDN-AWQ] CSDN VPTQ blog, section "02.02 AWQ": salient channels are found
  from the activation distribution; salient weight channels are scaled up by
  an equivalent transform whose scales come from offline activation
  statistics, with no backpropagation or reconstruction.

Readings where the pages are silent (each is also listed in the design notes):

* scale statistic: s_j = max(mean_i |x_ij|, 1e-8) ** alpha, alpha = 0.5,
  computed in float64 and stored as fp32 (no grid search, no normalisation);
* equivalent transform: w'_nk = fp16(fp32(W_nk) * s_k), x'_mk = fp16(fp32(x_mk) / s_k);
* group bounds lo/hi are the min/max of the folded group; the range is not
  forced to include 0;
* scale S = fp16(max(hi - lo, 1e-5) / 15) (fp32 subtract and divide), codes
  are computed against the stored fp16 S;
* zero z = clamp(rint(-lo / S), 0, 15), codes q = clamp(rint(w' / S) + z, 0, 15),
  rint = round half to even, fp32 division;
* dequantization ŵ = (q - z) * S, exact in float64; y = x' . ŵ^T in float64;
* scale search: an even grid of 20 exponents over [0, 1); the squared Frobenius
  error of the layer output on the calibration rows, against x . W^T, picks one;
* variants ([AWQ-README] model-zoo table INT3-g128; [AutoAWQ-blog] w_bit,
  q_group_size, zero_point): b-bit codes with qmax = 2^b - 1 in the same steps;
  zero_point false (symmetric): S = fp16(max(max |w'|, 1e-5) / (2^(b-1) - 1)),
  z = 2^(b-1) fixed, q = clamp(rint(w' / S) + z, 0, qmax); groups of 64 or 128.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``
(brute force, closed forms, invariants, exact rational arithmetic,
hand-derived golden fixtures). No function is "parity unpinned".
"""
from __future__ import annotations

from typing import Tuple

import numpy as np

BITS = 4
GROUP_SIZE = 128
QMAX = (1 << BITS) - 1          # 15
RANGE_FLOOR = np.float32(1e-5)  # floor on hi - lo (a constant group would divide by zero)
MEAN_FLOOR = 1e-8               # floor on the mean |x| before the power
K_TILE = 64                     # k per packed tile


# --------------------------------------------------------------------------
# a1: activation statistic and the activation side of the equivalent transform
# --------------------------------------------------------------------------
def activation_scale(x: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """Per-input-channel AWQ scale s[K] (fp32) from activations x[M, K] (fp16).

    [CSDN-AWQ] "02.02 AWQ": the scale of a channel comes from activation
    statistics. Reading: s_j = max(mean_i |x_ij|, 1e-8) ** alpha in float64,
    then rounded to fp32. For alpha = 0.5 the power is the square root (the
    same real number, correctly rounded).
    """
    x64 = np.abs(np.asarray(x, dtype=np.float16).astype(np.float64))
    mean = x64.sum(axis=0) / x64.shape[0]
    mean = np.maximum(mean, MEAN_FLOOR)
    a = float(np.float32(alpha))
    p = np.sqrt(mean) if a == 0.5 else np.power(mean, a)
    return p.astype(np.float32)


def scale_activations(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    """x'[M, K] = fp16(fp32(x) / s): the activation half of the equivalent transform.

    [CSDN-AWQ] "02.02 AWQ": salient weight channels are scaled up and the
    activations scaled down so that the product is unchanged.
    """
    xs = np.asarray(x, dtype=np.float16).astype(np.float32)
    return (xs / np.asarray(s, dtype=np.float32)[None, :]).astype(np.float16)


# --------------------------------------------------------------------------
# a2: fold + group quantizer
# --------------------------------------------------------------------------
def fold_weights(W: np.ndarray, s) -> np.ndarray:
    """w'[N, K] = fp16(fp32(W) * s_k): the weight half of the equivalent transform.

    ``s is None`` means no fold (w' = W).
    """
    W16 = np.asarray(W, dtype=np.float16)
    if s is None:
        return W16.copy()
    return (W16.astype(np.float32) * np.asarray(s, dtype=np.float32)[None, :]).astype(np.float16)


def quantize_groups(wf: np.ndarray) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Asymmetric 4-bit min/max quantization of w'[N, K] in groups of 128 along K.

    [AWQ-README] "Usage" (``--w_bit 4 --q_group_size 128``), [HF-AWQ] section 2
    (zero_point true, group_size 128, bits 4), [AutoAWQ-blog] (a group shares
    one scale and one zero point; zero_point selects asymmetric quantization).

    Returns codes q[N, K] (uint8, 0..15), scales S[N, K/128] (fp16) and zero
    points z[N, K/128] (uint8, 0..15).  Steps, per group, all fp32 round to
    nearest even:

    1. lo = min w', hi = max w'
    2. S = fp16(max(hi - lo, 1e-5) / 15)
    3. z = clamp(rint(-lo / S), 0, 15)
    4. q = clamp(rint(w' / S) + z, 0, 15)

    Min, max and clamp follow IEEE minNum/maxNum (a NaN operand is ignored),
    which is what CUDA's fminf/fmaxf do.
    """
    wf = np.asarray(wf, dtype=np.float16)
    N, K = wf.shape
    if K % GROUP_SIZE:
        raise ValueError("K must be a multiple of 128")
    G = K // GROUP_SIZE
    w = wf.astype(np.float32).reshape(N, G, GROUP_SIZE)
    lo = np.fmin.reduce(w, axis=2)
    hi = np.fmax.reduce(w, axis=2)
    rng = np.fmax(hi - lo, RANGE_FLOOR)
    S = (rng / np.float32(QMAX)).astype(np.float16)
    Sf = S.astype(np.float32)
    z = np.fmin(np.fmax(np.rint(-lo / Sf), np.float32(0)), np.float32(QMAX))
    q = np.rint(w / Sf[..., None]) + z[..., None]
    q = np.fmin(np.fmax(q, np.float32(0)), np.float32(QMAX))
    return q.astype(np.uint8).reshape(N, K), S, z.astype(np.uint8)


def quantize_groups_cfg(wf: np.ndarray, bits: int = BITS, group_size: int = GROUP_SIZE,
                        zero_point: bool = True) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """The quantizer for the configurations the pages name besides INT4-g128-asymmetric.

    [AWQ-README] model-zoo table (INT3-g128 models next to INT4-g128),
    [AutoAWQ-blog] "Quantizing a model with AutoAWQ" (``w_bit``, ``q_group_size``
    = the group that shares one scale and one zero point, ``zero_point`` =
    asymmetric quantization), [HF-AWQ] section 2 (bits, group_size, zero_point).

    Returns q[N, K] (uint8, 0..2^bits - 1), S[N, K/group] (fp16), z[N, K/group]
    (uint8). Per group, fp32 round to nearest even, with qmax = 2^bits - 1:

    * zero_point true (asymmetric): the steps of ``quantize_groups`` with 15
      replaced by qmax: S = fp16(max(hi - lo, 1e-5) / qmax),
      z = clamp(rint(-lo / S), 0, qmax);
    * zero_point false (symmetric): a = max(|lo|, |hi|),
      S = fp16(max(a, 1e-5) / (2^(bits-1) - 1)), z = 2^(bits-1): the signed
      code rint(w' / S) in [-2^(bits-1), 2^(bits-1) - 1] stored with the offset z;
    * q = clamp(rint(w' / S) + z, 0, qmax) in both cases.
    """
    if bits not in (3, 4) or group_size not in (64, 128):
        raise ValueError("bits must be 3 or 4 and group_size 64 or 128")
    wf = np.asarray(wf, dtype=np.float16)
    N, K = wf.shape
    if K % group_size:
        raise ValueError("K must be a multiple of the group size")
    qmax = np.float32((1 << bits) - 1)
    G = K // group_size
    w = wf.astype(np.float32).reshape(N, G, group_size)
    lo = np.fmin.reduce(w, axis=2)
    hi = np.fmax.reduce(w, axis=2)
    if zero_point:
        S = (np.fmax(hi - lo, RANGE_FLOOR) / qmax).astype(np.float16)
        Sf = S.astype(np.float32)
        z = np.fmin(np.fmax(np.rint(-lo / Sf), np.float32(0)), qmax)
    else:
        a = np.fmax(np.abs(lo), np.abs(hi))
        S = (np.fmax(a, RANGE_FLOOR) / np.float32((1 << (bits - 1)) - 1)).astype(np.float16)
        Sf = S.astype(np.float32)
        z = np.full(lo.shape, np.float32(1 << (bits - 1)))
    q = np.rint(w / Sf[..., None]) + z[..., None]
    q = np.fmin(np.fmax(q, np.float32(0)), qmax)
    return q.astype(np.uint8).reshape(N, K), S, z.astype(np.uint8)


def dequantize_cfg(q: np.ndarray, S: np.ndarray, z: np.ndarray, group_size: int) -> np.ndarray:
    """ŵ = (q - z) * S with groups of ``group_size`` along K, exact in float64."""
    N, K = q.shape
    G = K // group_size
    qg = q.astype(np.float64).reshape(N, G, group_size)
    w = (qg - z.astype(np.float64)[..., None]) * S.astype(np.float64)[..., None]
    return w.reshape(N, K)


def dequantize(q: np.ndarray, S: np.ndarray, z: np.ndarray) -> np.ndarray:
    """ŵ[N, K] = (q - z) * S in float64 (exact: a 5-bit integer times an fp16).

    [AWQ-README] "Usage" step 2: simulated ("fake") quantization is quantize
    then dequantize in floating point.
    """
    N, K = q.shape
    G = K // GROUP_SIZE
    qg = q.astype(np.float64).reshape(N, G, GROUP_SIZE)
    d = (qg - z.astype(np.float64)[..., None]) * S.astype(np.float64)[..., None]
    return d.reshape(N, K)


def fake_quantize(W: np.ndarray, s=None) -> np.ndarray:
    """dequantize(quantize(fold(W, s))) in float64."""
    return dequantize(*quantize_groups(fold_weights(W, s)))


# --------------------------------------------------------------------------
# a3/a4: the W4A16 linear layer
# --------------------------------------------------------------------------
def linear(xs: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """y[M, N] = x'[M, K] . ŵ[N, K]^T, float64 accumulation.

    [AWQ-README] "Installation" step 3: W4A16 kernels, 4-bit weights and
    16-bit activations; the layer is the ordinary linear map with the
    dequantized weight.
    """
    return np.asarray(xs, dtype=np.float16).astype(np.float64) @ np.asarray(w_hat, np.float64).T


def reference_forward(x: np.ndarray, W: np.ndarray, alpha: float = 0.5):
    """The whole path: s from x, fold, quantize, scale x, dequantize, matmul.

    Returns a dict with every intermediate.
    """
    s = activation_scale(x, alpha)
    xs = scale_activations(x, s)
    wf = fold_weights(W, s)
    q, S, z = quantize_groups(wf)
    y = linear(xs, dequantize(q, S, z))
    return {"s": s, "xs": xs, "wf": wf, "q": q, "S": S, "z": z, "y": y}


def check_tolerance(y: np.ndarray, y_ref: np.ndarray, rel_fro: float = 2e-3, max_rms: float = 1e-2):
    """The output bar: ||y - y_ref||_F / ||y_ref||_F <= 2e-3 and max|y - y_ref| <= 1e-2 rms(y_ref).

    Returns (ok, rel_fro_err, max_err / rms(y_ref)).
    """
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    diff = y - y_ref
    nref = np.linalg.norm(y_ref)
    rms = nref / np.sqrt(max(y_ref.size, 1))
    e_fro = float(np.linalg.norm(diff) / nref) if nref > 0 else float(np.linalg.norm(diff))
    e_max = float(np.max(np.abs(diff)) / rms) if rms > 0 and diff.size else float(np.max(np.abs(diff), initial=0.0))
    return (e_fro <= rel_fro and e_max <= max_rms), e_fro, e_max


# --------------------------------------------------------------------------
# Fused epilogues of the fused-N layers ("transformers - AWQ" section 3)
# --------------------------------------------------------------------------
def silu(v: np.ndarray) -> np.ndarray:
    """SiLU(v) = v / (1 + exp(-v)) in float64 (the Llama/Mistral MLP activation)."""
    v = np.asarray(v, np.float64)
    return v / (1.0 + np.exp(-v))


def gate_up_silu(y_gate_up: np.ndarray) -> np.ndarray:
    """h[M, I] = SiLU(y[:, :I]) * y[:, I:] for the fused gate+up output y[M, 2I] (gate rows first).

    [HF-AWQ] section 3: the fused MLP module takes the gate, up and down layers in that order;
    the gate/up pair of Llama and Mistral (the architectures the section names) combine as
    SiLU(gate) * up before the down projection. The pages print no activation; reading: SiLU.
    """
    y = np.asarray(y_gate_up, np.float64)
    I = y.shape[1] // 2
    return silu(y[:, :I]) * y[:, I:]


def split_qkv(y_qkv: np.ndarray, n_q: int, n_kv: int):
    """(q, k, v) = the column blocks [0, n_q), [n_q, n_q + n_kv), [n_q + n_kv, n_q + 2 n_kv) of the
    fused q/k/v output ([HF-AWQ] section 3: attention layers fused in the order query, key, value;
    num_key_value_heads < num_attention_heads gives the narrower k and v of grouped-query attention)."""
    y = np.asarray(y_qkv)
    return y[:, :n_q], y[:, n_q:n_q + n_kv], y[:, n_q + n_kv:n_q + 2 * n_kv]


# --------------------------------------------------------------------------
# AWQ scale search (the exponent alpha of the activation statistic)
# --------------------------------------------------------------------------
def alpha_grid(n_grid: int = 20) -> np.ndarray:
    """Candidate exponents alpha_i = i / n_grid, i = 0 .. n_grid - 1 (float32 values).

    [AWQ-README] "Usage" step 1 runs an AWQ search that picks the scales and
    dumps them; [CSDN-AWQ] "02.02 AWQ" says the scales come from offline
    activation statistics with no backpropagation. The pages give neither the
    grid nor its size; reading: an even grid over [0, 1) of 20 points.
    """
    return (np.arange(n_grid, dtype=np.float64) / n_grid).astype(np.float32)


def search_errors(x: np.ndarray, W: np.ndarray, alphas) -> np.ndarray:
    """Squared output error of the whole path for every candidate alpha, float64.

    For each alpha: s = activation_scale(x, alpha), x' = scale_activations(x, s),
    w_hat = dequantize(quantize_groups(fold_weights(W, s))), and
    err = || x . W^T - x' . w_hat^T ||_F^2 with both products in float64 over the
    fp16 inputs (the layer's own output on the calibration rows is the target).
    """
    y_ref = np.asarray(x, np.float16).astype(np.float64) @ np.asarray(W, np.float16).astype(np.float64).T
    errs = []
    for a in alphas:
        s = activation_scale(x, float(a))
        y = linear(scale_activations(x, s), fake_quantize(W, s))
        errs.append(float(np.sum((y - y_ref) ** 2)))
    return np.array(errs, dtype=np.float64)


def search_alpha(x: np.ndarray, W: np.ndarray, n_grid: int = 20):
    """The grid point with the smallest squared output error (the first one on ties).

    Returns (alpha, s, errors): the chosen exponent, its scale s[K] and the error of
    every grid point.
    """
    alphas = alpha_grid(n_grid)
    errs = search_errors(x, W, alphas)
    i = int(np.argmin(errs))
    return float(alphas[i]), activation_scale(x, float(alphas[i])), errs


# --------------------------------------------------------------------------
# Packed layout, version 2 (restated from its written specification)
# --------------------------------------------------------------------------
#
# Rows are grouped in 16-row tiles T (Ntiles = ceil(N / 16)); along K the
# groups are padded to an even count (G2 = ceil(G / 2) group pairs,
# KTp = 4 * G2 64-k tiles per tile).  Padding rows and padding groups hold
# code 0, scale 0 and zero 0.  Index names:
#   n = 16*T + 8*h + r                  (tile T, half h, row r)
#   k = 64*kt + 16*t + 4*s + 2*e1 + e0  (64-k tile kt, lane column t, step s, slot e)
#   g = k // 128
# qweight (uint32, Ntiles*KTp*128 words):
#   word   = (T*KTp + kt)*128 + (4*r + t)*4 + s
#   nibble = h + 2*e1 + 4*e0  (bits 4*nibble .. 4*nibble+3)
# scales (fp16, Ntiles*2*G2*16):  index (T*2*G2 + g)*16 + 2*r + h
# zeros  (uint8, Ntiles*2*G2*8):  byte  (T*2*G2 + g)*8 + r, low nibble h=0, high nibble h=1
# So every tile's codes, scales and zeros each run contiguously along K.
TILE_ROWS = 16


def layout_dims(N: int, K: int):
    """(Ntiles, G, G2, KTp) of an N x K layer."""
    G = K // GROUP_SIZE
    G2 = -(-G // 2)
    return -(-N // TILE_ROWS), G, G2, 4 * G2


def padded_rows(N: int) -> int:
    return layout_dims(N, GROUP_SIZE)[0] * TILE_ROWS


def pack(q: np.ndarray, S: np.ndarray, z: np.ndarray):
    """Codes/scales/zeros in plain [N, K] / [N, G] form -> (qweight, scales, zeros)."""
    N, K = q.shape
    NT, G, G2, KTp = layout_dims(N, K)
    qp = np.zeros((NT * TILE_ROWS, KTp * K_TILE), dtype=np.uint32)
    qp[:N, :K] = q
    # axes: T, h, r, kt, t, s, e1, e0
    a = qp.reshape(NT, 2, 8, KTp, 4, 4, 2, 2)
    # word order (T, kt, r, t, s); nibble order (e0, e1, h) -> nibble = 4*e0 + 2*e1 + h
    a = a.transpose(0, 3, 2, 4, 5, 7, 6, 1).reshape(-1, 8)
    shifts = (4 * np.arange(8)).astype(np.uint32)
    qweight = np.bitwise_or.reduce(a << shifts, axis=1).astype(np.uint32)

    Sp = np.zeros((NT * TILE_ROWS, 2 * G2), dtype=np.float16)
    Sp[:N, :G] = S
    scales = Sp.reshape(NT, 2, 8, 2 * G2).transpose(0, 3, 2, 1).reshape(-1).copy()   # T, g, r, h

    zp = np.zeros((NT * TILE_ROWS, 2 * G2), dtype=np.uint8)
    zp[:N, :G] = z
    zz = zp.reshape(NT, 2, 8, 2 * G2).transpose(0, 3, 2, 1)                          # T, g, r, h
    zeros = (zz[..., 0] | (zz[..., 1] << 4)).astype(np.uint8).reshape(-1)
    return qweight, scales, zeros


def unpack(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, N: int, K: int):
    """Inverse of ``pack``: (qweight, scales, zeros) -> (q[N, K], S[N, G], z[N, G])."""
    NT, G, G2, KTp = layout_dims(N, K)
    words = np.asarray(qweight, dtype=np.uint32).reshape(-1)
    if words.size != NT * KTp * 128:
        raise ValueError("qweight has the wrong size")
    shifts = (4 * np.arange(8)).astype(np.uint32)
    nib = ((words[:, None] >> shifts) & np.uint32(0xF)).astype(np.uint8)
    # nib axes: T, kt, r, t, s, e0, e1, h -> back to T, h, r, kt, t, s, e1, e0
    a = nib.reshape(NT, KTp, 8, 4, 4, 2, 2, 2).transpose(0, 7, 2, 1, 3, 4, 6, 5)
    q = a.reshape(NT * TILE_ROWS, KTp * K_TILE)[:N, :K].copy()

    sc = np.asarray(scales, dtype=np.float16).reshape(NT, 2 * G2, 8, 2)   # T, g, r, h
    S = sc.transpose(0, 3, 2, 1).reshape(NT * TILE_ROWS, 2 * G2)[:N, :G].copy()

    zb = np.asarray(zeros, dtype=np.uint8).reshape(NT, 2 * G2, 8)          # T, g, r
    zz = np.stack([zb & 0xF, zb >> 4], axis=-1)                           # T, g, r, h
    z = zz.transpose(0, 3, 2, 1).reshape(NT * TILE_ROWS, 2 * G2)[:N, :G].copy()
    return q, S, z


def packed_sizes(N: int, K: int):
    """(qweight words, scale halves, zero bytes) for an N x K layer."""
    NT, G, G2, KTp = layout_dims(N, K)
    return NT * KTp * 128, NT * 2 * G2 * 16, NT * 2 * G2 * 8
