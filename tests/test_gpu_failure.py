"""Failure detection on the GPU without a fault.

The prefill kernel bounds every mbarrier wait by %globaltimer. A test hook
shortens that bound to 1 ns, so the first wait that is not already satisfied
gives up on a healthy GPU. The kernel then records AWQ_ERR_TIMEOUT in the
device status word, drains its own copies and tensor-core work, frees its
tensor memory and returns. The host reads the status; the context stays
usable and the next call is correct.
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
