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
* dequantization ŵ = (q - z) * S, exact in float64; y = x' . ŵ^T in float64.

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
SUPER_ROWS = 128                # rows per super-tile of the packed layout
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
# Packed layout, version 1 (restated from its written specification)
# --------------------------------------------------------------------------
#
# Rows are padded to Np = ceil(N / 128) * 128; padding rows hold code 0,
# scale 0 and zero 0.  Index names:
#   n = st*128 + nt*16 + h*8 + r        (super-tile st, 16-row tile nt, half h, row r)
#   k = kt*64 + t*16 + s*4 + e1*2 + e0  (64-k tile kt, lane column t, step s, slot e)
#   g = k // 128
# qweight (uint32, Np*K/8 words):
#   word   = ((st*KT + kt)*8 + nt)*128 + (4*r + t)*4 + s,   KT = K/64
#   nibble = h + 2*e1 + 4*e0  (bits 4*nibble .. 4*nibble+3)
# scales (fp16, Np*K/128):  index ((st*G + g)*8 + nt)*16 + 2*r + h
# zeros  (uint8, Np*K/256): byte  ((st*G + g)*8 + nt)*8 + r, low nibble h=0, high nibble h=1
def padded_rows(N: int) -> int:
    return -(-N // SUPER_ROWS) * SUPER_ROWS


def pack(q: np.ndarray, S: np.ndarray, z: np.ndarray):
    """Codes/scales/zeros in plain [N, K] / [N, G] form -> (qweight, scales, zeros)."""
    N, K = q.shape
    G = K // GROUP_SIZE
    Np = padded_rows(N)
    ST, KT = Np // SUPER_ROWS, K // K_TILE
    qp = np.zeros((Np, K), dtype=np.uint32)
    qp[:N] = q
    # axes: st, nt, h, r, kt, t, s, e1, e0
    a = qp.reshape(ST, 8, 2, 8, KT, 4, 4, 2, 2)
    # word order (st, kt, nt, r, t, s); nibble order (e0, e1, h) -> nibble = 4*e0 + 2*e1 + h
    a = a.transpose(0, 4, 1, 3, 5, 6, 8, 7, 2).reshape(-1, 8)
    shifts = (4 * np.arange(8)).astype(np.uint32)
    qweight = np.bitwise_or.reduce(a << shifts, axis=1).astype(np.uint32)

    Sp = np.zeros((Np, G), dtype=np.float16)
    Sp[:N] = S
    scales = Sp.reshape(ST, 8, 2, 8, G).transpose(0, 4, 1, 3, 2).reshape(-1).copy()

    zp = np.zeros((Np, G), dtype=np.uint8)
    zp[:N] = z
    zz = zp.reshape(ST, 8, 2, 8, G).transpose(0, 4, 1, 3, 2)   # st, g, nt, r, h
    zeros = (zz[..., 0] | (zz[..., 1] << 4)).astype(np.uint8).reshape(-1)
    return qweight, scales, zeros


def unpack(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, N: int, K: int):
    """Inverse of ``pack``: (qweight, scales, zeros) -> (q[N, K], S[N, G], z[N, G])."""
    G = K // GROUP_SIZE
    Np = padded_rows(N)
    ST, KT = Np // SUPER_ROWS, K // K_TILE
    words = np.asarray(qweight, dtype=np.uint32).reshape(-1)
    if words.size != Np * K // 8:
        raise ValueError("qweight has the wrong size")
    shifts = (4 * np.arange(8)).astype(np.uint32)
    nib = ((words[:, None] >> shifts) & np.uint32(0xF)).astype(np.uint8)
    # nib axes: st, kt, nt, r, t, s, e0, e1, h -> back to st, nt, h, r, kt, t, s, e1, e0
    a = nib.reshape(ST, KT, 8, 8, 4, 4, 2, 2, 2).transpose(0, 2, 8, 3, 1, 4, 5, 7, 6)
    q = a.reshape(Np, K)[:N].copy()

    sc = np.asarray(scales, dtype=np.float16).reshape(ST, G, 8, 8, 2)  # st, g, nt, r, h
    S = sc.transpose(0, 2, 4, 3, 1).reshape(Np, G)[:N].copy()

    zb = np.asarray(zeros, dtype=np.uint8).reshape(ST, G, 8, 8)         # st, g, nt, r
    zz = np.stack([zb & 0xF, zb >> 4], axis=-1)                        # st, g, nt, r, h
    z = zz.transpose(0, 2, 4, 3, 1).reshape(Np, G)[:N].copy()
    return q, S, z


def packed_sizes(N: int, K: int):
    """(qweight words, scale halves, zero bytes) for an N x K layer."""
    Np = padded_rows(N)
    return Np * K // 8, Np * K // GROUP_SIZE, Np * K // (2 * GROUP_SIZE)
