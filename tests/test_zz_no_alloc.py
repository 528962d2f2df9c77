"""The scale search without a caller workspace (awq_search_alpha_noalloc).

Its scratch is a fixed array in the library's device memory shared by every call, so the GPU
test runs two searches of different shapes back to back and checks each against
awq_search_alpha on a workspace of its own. The search's reduction order is fixed, so the two
entry points must agree bit for bit (the reproducibility bar of the other search tests).
This file is collected last so that the shared array has already served other kernels' callers
when the suite runs as a whole; it passes alone as well.
"""
import ctypes

import numpy as np
import pytest

import workloads
from gpu_util import dev, host, lib, torch_mod

V = ctypes.c_void_p
ALPHAS = [i / 20.0 for i in range(20)]


def _call_noalloc(P, x, W, alphas):
    """One call through the C-ABI; returns (status, err, best) with the outputs pre-filled."""
    torch = torch_mod()
    M, K = x.shape
    N = W.shape[0]
    a = (ctypes.c_float * len(alphas))(*alphas)
    err = torch.full((len(alphas),), float("nan"), dtype=torch.float64, device=x.device)
    best = torch.full((1,), -1, dtype=torch.int32, device=x.device)
    st = P.load_library().awq_search_alpha_noalloc(V(x.data_ptr()), V(W.data_ptr()), M, N, K,
                                                    ctypes.cast(a, V), len(alphas), V(err.data_ptr()),
                                                    V(best.data_ptr()), V(torch.cuda.current_stream().cuda_stream))
    return st, err, best


def test_noalloc_limit_matches_the_workspace_size():
    """Host-side check (no GPU): shapes past the fixed scratch are refused before any CUDA call."""
    P = lib()
    L = P.load_library()
    assert P.SEARCH_NOALLOC_SCRATCH_BYTES == 64 << 20
    assert L.awq_search_workspace_bytes(1781, 4096, 4096) <= P.SEARCH_NOALLOC_SCRATCH_BYTES
    assert L.awq_search_workspace_bytes(1782, 4096, 4096) > P.SEARCH_NOALLOC_SCRATCH_BYTES
    assert L.awq_search_workspace_bytes(492, 8192, 8192) > P.SEARCH_NOALLOC_SCRATCH_BYTES
    a = (ctypes.c_float * 1)(0.5)
    st = L.awq_search_alpha_noalloc(V(16), V(16), 1782, 4096, 4096, ctypes.cast(a, V), 1, V(16), V(16), None)
    assert st == P.AWQ_ERR_INVALID_ARG


@pytest.mark.gpu
def test_noalloc_search_equals_the_workspace_search_on_two_calls_in_a_row():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    P = lib()
    cases = [workloads.random_case(131, 48, 200, 1280), workloads.random_case(137, 4, 64, 512)]
    inputs = [(dev(x), dev(W)) for x, W in cases]
    refs = []
    for x, W in inputs:
        err, best, _ = P.awq_search_alpha(x, W, ALPHAS)
        refs.append((host(err), int(host(best)[0])))

    # two calls in a row on the shared scratch, the second on a smaller shape
    outs = [_call_noalloc(P, x, W, ALPHAS) for x, W in inputs]
    torch.cuda.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK
    for (st, err, best), (e_ref, b_ref) in zip(outs, refs):
        assert st == P.AWQ_OK, P.status_string(st)
        e = host(err)
        assert np.all(np.isfinite(e))
        assert np.array_equal(e, e_ref), (e, e_ref)
        assert int(host(best)[0]) == b_ref

    # a shape past the fixed scratch is refused and leaves the outputs alone
    xb = torch.zeros((1782, 4096), dtype=torch.float16, device="cuda")
    Wb = torch.zeros((4096, 4096), dtype=torch.float16, device="cuda")
    st, err, best = _call_noalloc(P, xb, Wb, ALPHAS[:2])
    torch.cuda.synchronize()
    assert st == P.AWQ_ERR_INVALID_ARG
    assert np.all(np.isnan(host(err))) and int(host(best)[0]) == -1
