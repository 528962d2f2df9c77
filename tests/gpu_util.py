"""Helpers for the GPU parity tests: move seeded inputs to the device, run the
library, and build oracle expectations (the oracle only ever sees the seeded
inputs, never a CUDA result)."""
import numpy as np

from oracle import awq_oracle as O


def torch_mod():
    import torch
    return torch


def dev(a: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def lib():
    import weight_only_quantization_w4a16_b200 as P
    P.load_library()
    return P


def oracle_packed(W: np.ndarray, s):
    """Oracle codes for W (folded with s) packed to layout v2 (numpy arrays)."""
    q, S, z = O.quantize_groups(O.fold_weights(W, s))
    return O.pack(q, S, z), (q, S, z)


def upload_packed(packed):
    qw, sc, zb = packed
    return dev(qw.view(np.int32)), dev(sc), dev(zb)


def f16_bits(a):
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def assert_tolerance(y, y_ref, what=""):
    ok, ef, em = O.check_tolerance(y, y_ref)
    assert ok, f"{what}: rel Frobenius {ef:.3e} (bar 2e-3), max/rms {em:.3e} (bar 1e-2)"
    return ef, em


def assert_tight(y, y_ref, rel=2.0 ** -10, abs_rms=1e-3, what=""):
    """A bound well inside the official bar: fp16 output rounding plus a small accumulation term."""
    y = np.asarray(y, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    rms = np.sqrt(np.mean(y_ref ** 2))
    err = np.abs(y - y_ref)
    bound = rel * np.abs(y_ref) + abs_rms * rms
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond the tight bound; worst {np.max(err - bound):.3e}"
