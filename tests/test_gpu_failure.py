"""Failure detection on the GPU without a fault.

Every kernel bounds its mbarrier waits by %globaltimer. One test hook
shortens that bound to 1 ns, so a wait that is not already satisfied gives up
on a healthy GPU (the prefill kernel's long accumulator waits always are).
A second hook makes the producer of the quantizer and of the decode kernels
skip the copies of its first pipeline stage: a wait on a phase that nothing
will ever complete, which can only end by running out its budget. The kernel
then records AWQ_ERR_TIMEOUT in the device status word, drains its own copies
(and tensor-core work, and frees its tensor memory) and returns. The host
reads the status; the context stays usable and the next call is correct.
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


def _with_lost_copy(P, call):
    """Runs `call` with the first stage's copies dropped and a 1 ns wait budget; returns the status."""
    P.awq_debug_set_wait_budget_ns(1)
    P.awq_debug_drop_first_copy(True)
    try:
        call()
        status = P.awq_poll_device_status()
    finally:
        P.awq_debug_drop_first_copy(False)
        P.awq_debug_set_wait_budget_ns(0)
    return status


def test_prefill_wait_budget_runs_out_then_recovers():
    P = lib()
    torch = torch_mod()
    M, N, K = 300, 1024, 4096
    x, W = workloads.random_case(81, M, N, K)
    r = O.reference_forward(x, W)
    s, xs = P.awq_activation_scale(dev(x))
    qw, sc, zb = P.awq_quantize_g128(dev(W), s)
    torch.cuda.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK

    P.awq_debug_set_wait_budget_ns(1)
    try:
        P.awq_w4a16_gemm(xs, qw, sc, zb, N)
        status = P.awq_poll_device_status()
    finally:
        P.awq_debug_set_wait_budget_ns(0)
    assert status == P.AWQ_ERR_TIMEOUT

    # the status is cleared by the poll; the context still works and results are right again
    assert P.awq_poll_device_status() == P.AWQ_OK
    y = P.awq_w4a16_gemm(xs, qw, sc, zb, N)
    assert P.awq_poll_device_status() == P.AWQ_OK
    assert_tolerance(host(y).astype(np.float64), r["y"], "gemm after a timeout")


def test_decode_and_quantizer_lost_copy_then_recover():
    """The cluster decode kernel and the quantizer give up on a stage whose copies never came."""
    P = lib()
    torch = torch_mod()
    M, N, K = 8, 1000, 2304
    x, W = workloads.random_case(85, M, N, K)
    r = O.reference_forward(x, W)
    s, xs = P.awq_activation_scale(dev(x))
    Wd = dev(W)
    torch.cuda.synchronize()
    assert P.awq_poll_device_status() == P.AWQ_OK

    assert _with_lost_copy(P, lambda: P.awq_quantize_g128(Wd, s)) == P.AWQ_ERR_TIMEOUT
    qw, sc, zb = P.awq_quantize_g128(Wd, s)
    assert P.awq_poll_device_status() == P.AWQ_OK
    q_ref = O.pack(r["q"], r["S"], r["z"])
    assert np.array_equal(host(qw).view(np.uint32), q_ref[0])

    assert _with_lost_copy(P, lambda: P.awq_w4a16_gemv(xs, qw, sc, zb, N)) == P.AWQ_ERR_TIMEOUT
    y = P.awq_w4a16_gemv(xs, qw, sc, zb, N)
    assert P.awq_poll_device_status() == P.AWQ_OK
    assert_tolerance(host(y).astype(np.float64), r["y"], "gemv after a timeout")
