"""AWQ W4A16 g128 for NVIDIA B200 — Python binding of ``libawq_w4a16.so``.

The binding only marshals arguments: it checks tensor dtypes, shapes and
devices, allocates outputs with PyTorch when the caller gives none, and
passes raw device pointers plus the current CUDA stream to the C ABI declared
in ``include/awq_w4a16.h``. Every step of the path runs in the library's
CUDA kernels; if the library is missing, every call raises.

Functions (same names as the C ABI):

* ``awq_activation_scale(x, alpha)``  -> (s[K] fp32, x'[M,K] fp16)
* ``awq_scale_activations(x, s)`` -> x'[M,K] fp16 with a stored s
* ``awq_quantize_g128(W, fold_scale)`` -> (qweight int32, scales fp16, zeros uint8)
* ``awq_w4a16_gemv(x, qweight, scales, zeros, N)`` -> y[M,N] fp16 (M <= 32)
* ``awq_w4a16_gemm(x, qweight, scales, zeros, N)`` -> y[M,N] fp16
* ``awq_w4a16_linear(...)``: gemv for M <= 32, gemm otherwise
* ``awq_w4a16_linear_qkv(x, qweight, scales, zeros, Nq, Nkv)`` -> (q, k, v): fused q/k/v split
* ``awq_w4a16_linear_silu_mul(x, qweight, scales, zeros, I)`` -> h = SiLU(gate) * up
* ``awq_search_alpha(x, W, alphas)`` -> (err[n] float64, best index): the AWQ scale search
* ``awq_poll_device_status()``, test hooks ``awq_debug_set_wait_budget_ns(ns)``,
  ``awq_debug_drop_first_copy(enable)``, ``awq_debug_set_gemm_split(ks)``
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libawq_w4a16.so")

AWQ_OK = 0
AWQ_ERR_INVALID_ARG = 1
AWQ_ERR_UNSUPPORTED = 2
AWQ_ERR_MISALIGNED = 3
AWQ_ERR_CUDA = 4
AWQ_ERR_TIMEOUT = 5
AWQ_ERR_BOUNDS = 6    # debug builds only

GROUP_SIZE = 128
BITS = 4

_lib = None


class AWQError(RuntimeError):
    """A C-ABI call returned a status other than AWQ_OK."""

    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg}")
        self.status = status


_VP = ctypes.c_void_p
_I = ctypes.c_int
_SIGS = {
    "awq_layout_version": ([], ctypes.c_int),
    "awq_status_string": ([_I], ctypes.c_char_p),
    "awq_check_config": ([_I, _I, _I], _I),
    "awq_qweight_bytes": ([_I, _I], ctypes.c_size_t),
    "awq_scales_bytes": ([_I, _I], ctypes.c_size_t),
    "awq_zeros_bytes": ([_I, _I], ctypes.c_size_t),
    "awq_activation_scale": ([_VP, _I, _I, ctypes.c_float, _VP, _VP, _VP], _I),
    "awq_scale_activations": ([_VP, _VP, _I, _I, _VP, _VP], _I),
    "awq_quantize_g128": ([_VP, _VP, _I, _I, _VP, _VP, _VP, _VP], _I),
    "awq_quantize": ([_VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP], _I),
    "awq_w4a16_gemv": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP], _I),
    "awq_w4a16_gemm": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP], _I),
    "awq_w4a16_linear": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP], _I),
    "awq_poll_device_status": ([_VP], _I),
    "awq_search_workspace_bytes": ([_I, _I, _I], ctypes.c_size_t),
    "awq_w4a16_linear_qkv": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP], _I),
    "awq_w4a16_linear_silu_mul": ([_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _VP], _I),
    "awq_search_alpha": ([_VP, _VP, _I, _I, _I, _VP, _I, _VP, _VP, _VP, ctypes.c_size_t, _VP], _I),
    "awq_search_alpha_noalloc": ([_VP, _VP, _I, _I, _I, _VP, _I, _VP, _VP, _VP], _I),
    "awq_debug_set_wait_budget_ns": ([ctypes.c_ulonglong], _I),
    "awq_debug_drop_first_copy": ([_I], _I),
    "awq_debug_set_gemm_split": ([_I], _I),
    "awq_gemm_plan": ([_I, _I, _I, _I, _I, ctypes.POINTER(_I), ctypes.POINTER(_I), ctypes.POINTER(ctypes.c_longlong)],
                      _I),
}


def library_path() -> str:
    return LIB_PATH


def load_library(path: Optional[str] = None):
    """Loads libawq_w4a16.so (built in-tree by ``build.py``). Raises if absent."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError(
            f"{p} is missing: build it with `python -m weight_only_quantization_w4a16_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(p)
    for name, (args, res) in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load_library().awq_status_string(int(status)).decode()


def _check(fn: str, status: int):
    if status != AWQ_OK:
        raise AWQError(fn, status, status_string(status))


LAYOUT_VERSION = 2   # the packed-weight layout this binding's size checks assume


def layout_version() -> int:
    return int(load_library().awq_layout_version())


def check_config(bits: int, group_size: int, zero_point: bool) -> bool:
    return load_library().awq_check_config(int(bits), int(group_size), int(bool(zero_point))) == AWQ_OK


def packed_nbytes(N: int, K: int) -> Tuple[int, int, int]:
    lib = load_library()
    return (int(lib.awq_qweight_bytes(N, K)), int(lib.awq_scales_bytes(N, K)), int(lib.awq_zeros_bytes(N, K)))


# ---------------------------------------------------------------------------- torch marshalling
def _torch():
    import torch
    return torch


def _stream_ptr():
    torch = _torch()
    return _VP(torch.cuda.current_stream().cuda_stream)


def _ptr(t) -> _VP:
    return _VP(t.data_ptr()) if t is not None else _VP(0)


def _need(t, dtype, name, dims=None, require_cuda=True):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if require_cuda:
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.device.index != torch.cuda.current_device():
            raise ValueError(f"{name} is on {t.device}, but the current CUDA device is "
                             f"cuda:{torch.cuda.current_device()} (the library runs on the current device)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dims is not None and t.dim() != dims:
        raise ValueError(f"{name} must have {dims} dimensions")


def _packed_sizes_host(N: int, K: int) -> Tuple[int, int, int]:
    """Byte sizes of packed layout v2 computed here (used before a library call, so that a caller's
    buffers are checked against the same figures the library states)."""
    if N < 1 or K < GROUP_SIZE or K % GROUP_SIZE:
        return 0, 0, 0
    tiles, pairs = -(-N // 16), -(-(K // GROUP_SIZE) // 2)
    return tiles * pairs * 2048, tiles * pairs * 64, tiles * pairs * 16


def _check_packed(qweight, scales, zeros, N: int, K: int, require_cuda=True):
    torch = _torch()
    _need(qweight, torch.int32, "qweight", require_cuda=require_cuda)
    _need(scales, torch.float16, "scales", require_cuda=require_cuda)
    _need(zeros, torch.uint8, "zeros", require_cuda=require_cuda)
    qb, sb, zb = _packed_sizes_host(N, K)
    if qb == 0:
        raise ValueError("N >= 1 and K a positive multiple of 128 are required")
    if qweight.numel() * 4 < qb or scales.numel() * 2 < sb or zeros.numel() < zb:
        raise ValueError(f"packed weight tensors are too small for N={N}, K={K}: need {qb}, {sb}, {zb} bytes")


def _check_vec(v, K: int, name: str, require_cuda=True):
    torch = _torch()
    _need(v, torch.float32, name, 1, require_cuda=require_cuda)
    if v.numel() != K:
        raise ValueError(f"{name} must have K={K} elements, got {v.numel()}")


def validate_activation_scale(x, s_out, x_scaled, require_cuda=True):
    torch = _torch()
    _need(x, torch.float16, "x", 2, require_cuda=require_cuda)
    M, K = x.shape
    _check_vec(s_out, K, "s_out", require_cuda)
    if x_scaled is not None:
        _need(x_scaled, torch.float16, "x_scaled", 2, require_cuda=require_cuda)
        if tuple(x_scaled.shape) != (M, K):
            raise ValueError(f"x_scaled must have shape {(M, K)}, got {tuple(x_scaled.shape)}")


def validate_scale_activations(x, s, x_scaled, require_cuda=True):
    torch = _torch()
    _need(x, torch.float16, "x", 2, require_cuda=require_cuda)
    M, K = x.shape
    _check_vec(s, K, "s", require_cuda)
    _need(x_scaled, torch.float16, "x_scaled", 2, require_cuda=require_cuda)
    if tuple(x_scaled.shape) != (M, K):
        raise ValueError(f"x_scaled must have shape {(M, K)}, got {tuple(x_scaled.shape)}")


def validate_quantize(W, fold_scale, out, require_cuda=True):
    torch = _torch()
    _need(W, torch.float16, "W", 2, require_cuda=require_cuda)
    N, K = W.shape
    if fold_scale is not None:
        _check_vec(fold_scale, K, "fold_scale", require_cuda)
    _check_packed(*out, N, K, require_cuda=require_cuda)


def validate_linear(x, qweight, scales, zeros, N: int, y, require_cuda=True):
    torch = _torch()
    _need(x, torch.float16, "x", 2, require_cuda=require_cuda)
    M, K = x.shape
    _check_packed(qweight, scales, zeros, N, K, require_cuda=require_cuda)
    _need(y, torch.float16, "y", 2, require_cuda=require_cuda)
    if tuple(y.shape) != (M, N):
        raise ValueError(f"y must have shape {(M, N)}, got {tuple(y.shape)}")


def awq_activation_scale(x, alpha: float = 0.5, s_out=None, x_scaled=None, want_scaled: bool = True):
    """a1: s[K] = max(mean_m |x[m,k]|, 1e-8)^alpha and x' = fp16(x / s)."""
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    if s_out is None:
        s_out = torch.empty(K, dtype=torch.float32, device=x.device)
    if want_scaled and x_scaled is None:
        x_scaled = torch.empty_like(x)
    validate_activation_scale(x, s_out, x_scaled)
    st = load_library().awq_activation_scale(_ptr(x), M, K, float(alpha), _ptr(s_out), _ptr(x_scaled),
                                             _stream_ptr())
    _check("awq_activation_scale", st)
    return s_out, x_scaled


def alloc_packed(N: int, K: int, device="cuda"):
    """Output tensors for awq_quantize_g128: qweight (int32 words), scales (fp16), zeros (uint8)."""
    torch = _torch()
    qb, sb, zb = packed_nbytes(N, K)
    if qb == 0:
        raise ValueError("N >= 1 and K a positive multiple of 128 are required")
    return (torch.empty(qb // 4, dtype=torch.int32, device=device),
            torch.empty(sb // 2, dtype=torch.float16, device=device),
            torch.empty(zb, dtype=torch.uint8, device=device))


def awq_quantize_g128(W, fold_scale=None, out=None):
    """a2: fold s into W[N,K] and quantize to packed layout v2. Returns (qweight, scales, zeros)."""
    torch = _torch()
    _need(W, torch.float16, "W", 2)
    N, K = W.shape
    out = out if out is not None else alloc_packed(N, K, W.device)
    validate_quantize(W, fold_scale, out)
    qweight, scales, zeros = out
    st = load_library().awq_quantize_g128(_ptr(W), _ptr(fold_scale), N, K, _ptr(qweight), _ptr(scales),
                                          _ptr(zeros), _stream_ptr())
    _check("awq_quantize_g128", st)
    return qweight, scales, zeros


def awq_quantize(W, fold_scale=None, bits: int = 4, group_size: int = 128, zero_point: bool = True, out=None):
    """a2 variants: INT4 or INT3 codes, asymmetric (zero_point) or symmetric, group size 128, in
    packed layout v2. Returns (qweight, scales, zeros)."""
    torch = _torch()
    _need(W, torch.float16, "W", 2)
    N, K = W.shape
    out = out if out is not None else alloc_packed(N, K, W.device)
    validate_quantize(W, fold_scale, out)
    qweight, scales, zeros = out
    st = load_library().awq_quantize(_ptr(W), _ptr(fold_scale), N, K, int(bits), int(group_size), int(bool(zero_point)),
                                     _ptr(qweight), _ptr(scales), _ptr(zeros), _stream_ptr())
    _check("awq_quantize", st)
    return qweight, scales, zeros


def _linear(fn_name: str, x, qweight, scales, zeros, N: int, y=None):
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    if y is None:
        y = torch.empty((M, N), dtype=torch.float16, device=x.device)
    validate_linear(x, qweight, scales, zeros, N, y)
    st = getattr(load_library(), fn_name)(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(y), M, N, K,
                                          _stream_ptr())
    _check(fn_name, st)
    return y


def awq_w4a16_gemv(x, qweight, scales, zeros, N: int, y=None):
    """a3: y[M,N] = x' . dequant^T for M <= 32 (decode)."""
    return _linear("awq_w4a16_gemv", x, qweight, scales, zeros, N, y)


def awq_w4a16_gemm(x, qweight, scales, zeros, N: int, y=None):
    """a4: y[M,N] = x' . dequant^T on tcgen05 tensor cores (prefill)."""
    return _linear("awq_w4a16_gemm", x, qweight, scales, zeros, N, y)


def awq_w4a16_linear(x, qweight, scales, zeros, N: int, y=None):
    """The decode kernel for small M, the prefill kernel otherwise (the library picks)."""
    return _linear("awq_w4a16_linear", x, qweight, scales, zeros, N, y)


def awq_w4a16_linear_qkv(x, qweight, scales, zeros, Nq: int, Nkv: int, out=None):
    """Fused q/k/v layer (weight rows: Nq query, Nkv key, Nkv value); returns (q, k, v)."""
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    N = Nq + 2 * Nkv
    if out is None:
        out = tuple(torch.empty((M, n), dtype=torch.float16, device=x.device) for n in (Nq, Nkv, Nkv))
    _check_packed(qweight, scales, zeros, N, K)
    for t, n, name in zip(out, (Nq, Nkv, Nkv), ("q", "k", "v")):
        _need(t, torch.float16, name, 2)
        if tuple(t.shape) != (M, n):
            raise ValueError(f"{name} must have shape {(M, n)}")
    st = load_library().awq_w4a16_linear_qkv(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), *[_ptr(t) for t in out],
                                             M, Nq, Nkv, K, _stream_ptr())
    _check("awq_w4a16_linear_qkv", st)
    return out


def awq_w4a16_linear_silu_mul(x, qweight, scales, zeros, I: int, h=None):
    """Fused gate+up layer (weight rows: I gate, then I up; I % 16 == 0): h = SiLU(gate) * up."""
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    if I < 16 or I % 16:
        raise ValueError("I must be a positive multiple of 16")
    if h is None:
        h = torch.empty((M, I), dtype=torch.float16, device=x.device)
    _check_packed(qweight, scales, zeros, 2 * I, K)
    _need(h, torch.float16, "h", 2)
    if tuple(h.shape) != (M, I):
        raise ValueError(f"h must have shape {(M, I)}")
    st = load_library().awq_w4a16_linear_silu_mul(_ptr(x), _ptr(qweight), _ptr(scales), _ptr(zeros), _ptr(h), M, I,
                                                  K, _stream_ptr())
    _check("awq_w4a16_linear_silu_mul", st)
    return h


def awq_search_alpha(x, W, alphas=None, workspace=None):
    """AWQ scale search: the squared output error of the whole path for every candidate exponent.

    ``alphas`` defaults to an even grid of 20 points over [0, 1). Returns (err, best, alphas) with
    err a float64 CUDA tensor and best a one-element int32 CUDA tensor (no host synchronization).
    """
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    _need(W, torch.float16, "W", 2)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError(f"W must have K={K} columns")
    if alphas is None:
        alphas = [i / 20.0 for i in range(20)]
    a = (ctypes.c_float * len(alphas))(*[float(v) for v in alphas])
    lib = load_library()
    need = int(lib.awq_search_workspace_bytes(M, N, K))
    if need == 0:
        raise ValueError("shape out of range for the search")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    _need(workspace, torch.uint8, "workspace", 1)
    if workspace.numel() < need:
        raise ValueError(f"workspace must hold {need} bytes")
    err = torch.empty(len(alphas), dtype=torch.float64, device=x.device)
    best = torch.empty(1, dtype=torch.int32, device=x.device)
    st = lib.awq_search_alpha(_ptr(x), _ptr(W), M, N, K, ctypes.cast(a, _VP), len(alphas), _ptr(err), _ptr(best),
                              _ptr(workspace), workspace.numel(), _stream_ptr())
    _check("awq_search_alpha", st)
    return err, best, list(alphas)


SEARCH_NOALLOC_SCRATCH_BYTES = 64 << 20   # the fixed scratch of awq_search_alpha_noalloc


def awq_search_alpha_noalloc(x, W, alphas=None):
    """The scale search on the library's fixed device scratch (no workspace argument).

    For callers that cannot allocate device memory themselves; results equal awq_search_alpha's.
    Shapes whose workspace would exceed SEARCH_NOALLOC_SCRATCH_BYTES raise ValueError. Only the
    outputs err and best are allocated here, by the caller's framework.
    """
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    _need(W, torch.float16, "W", 2)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError(f"W must have K={K} columns")
    if alphas is None:
        alphas = [i / 20.0 for i in range(20)]
    a = (ctypes.c_float * len(alphas))(*[float(v) for v in alphas])
    lib = load_library()
    need = int(lib.awq_search_workspace_bytes(M, N, K))
    if need == 0 or need > SEARCH_NOALLOC_SCRATCH_BYTES:
        raise ValueError(f"shape out of range for the search without workspace ({need} bytes needed)")
    err = torch.empty(len(alphas), dtype=torch.float64, device=x.device)
    best = torch.empty(1, dtype=torch.int32, device=x.device)
    st = lib.awq_search_alpha_noalloc(_ptr(x), _ptr(W), M, N, K, ctypes.cast(a, _VP), len(alphas), _ptr(err),
                                      _ptr(best), _stream_ptr())
    _check("awq_search_alpha_noalloc", st)
    return err, best, list(alphas)


def awq_poll_device_status() -> int:
    """Synchronizes the current stream and returns (and clears) the device status code."""
    return int(load_library().awq_poll_device_status(_stream_ptr()))


def awq_debug_set_wait_budget_ns(ns: int) -> None:
    _check("awq_debug_set_wait_budget_ns", load_library().awq_debug_set_wait_budget_ns(int(ns)))


def awq_debug_drop_first_copy(enable: bool) -> None:
    _check("awq_debug_drop_first_copy", load_library().awq_debug_drop_first_copy(int(bool(enable))))


def awq_gemm_plan(M: int, N: int, K: int, epilogue: int = 0, num_sms: Optional[int] = None) -> Tuple[int, int, int]:
    """(token tile, K split, split tiles) that the prefill kernel takes for this shape (host-only).
    epilogue: 0 plain, 1 q/k/v split, 2 gate/up SiLU*up; num_sms defaults to the current device's."""
    if num_sms is None:
        import torch
        num_sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    bt, ks, nsplit = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_longlong(0)
    _check("awq_gemm_plan", load_library().awq_gemm_plan(int(M), int(N), int(K), int(epilogue), int(num_sms),
                                                          ctypes.byref(bt), ctypes.byref(ks), ctypes.byref(nsplit)))
    return bt.value, ks.value, nsplit.value


def awq_debug_set_gemm_split(ks: int) -> None:
    """Prefill K split: 0 chooses per launch, 1 never splits, 2 splits every tile across a CTA pair,
    3 the mixed form (whole rounds, then the rest split) on a grid of 3 CTA pairs (a test form)."""
    _check("awq_debug_set_gemm_split", load_library().awq_debug_set_gemm_split(int(ks)))


class AWQLinear:
    """A quantized linear layer: packed weights plus the per-channel fold scale.

    ``AWQLinear.from_float(W, x_calib)`` runs the whole path on the GPU: the
    activation statistic of ``x_calib`` (a1), the fold and quantizer (a2);
    ``layer(x)`` scales the activations by 1/s and runs the W4A16 kernel
    (a3 for M <= 32, a4 otherwise).
    """

    def __init__(self, qweight, scales, zeros, s, N: int, K: int):
        self.qweight, self.scales, self.zeros, self.s = qweight, scales, zeros, s
        self.N, self.K = N, K

    @classmethod
    def from_float(cls, W, x_calib, alpha: float = 0.5):
        s, _ = awq_activation_scale(x_calib, alpha, want_scaled=False)
        q, sc, z = awq_quantize_g128(W, s)
        return cls(q, sc, z, s, W.shape[0], W.shape[1])

    def __call__(self, x, y=None):
        xs = awq_scale_activations(x, self.s)
        return awq_w4a16_linear(xs, self.qweight, self.scales, self.zeros, self.N, y)


def awq_scale_activations(x, s, x_scaled=None):
    """a1 with a stored s: x' = fp16(x / s) (the activation half of the equivalent transform)."""
    torch = _torch()
    _need(x, torch.float16, "x", 2)
    M, K = x.shape
    if x_scaled is None:
        x_scaled = torch.empty_like(x)
    validate_scale_activations(x, s, x_scaled)
    st = load_library().awq_scale_activations(_ptr(x), _ptr(s), M, K, _ptr(x_scaled), _stream_ptr())
    _check("awq_scale_activations", st)
    return x_scaled
