"""GPU parity of the AWQ scale search against the oracle's search.

The GPU scores each candidate with the library's own path (fp16 layer output), the
oracle in float64, so the errors agree to the output rounding; the chosen exponent is
compared where the oracle's best and second best are further apart than that.
"""
import numpy as np
import pytest

from oracle import awq_oracle as O
import workloads
from gpu_util import dev, host, lib, torch_mod

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = torch_mod()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib()


def _known_optimum_case(seed=5, M=8, N=32, K=256):
    rng = np.random.default_rng(seed)
    k = np.array([-1, 0, 1, 2] * (K // 4))
    x = (np.where(rng.random((M, K)) < 0.5, -1.0, 1.0) * (4.0 ** k)[None, :]).astype(np.float16)
    m = rng.integers(0, 16, (N, K))
    m[:, 0::128] = 0
    m[:, 1::128] = 15
    W = (m * 2.0 ** (-6 - k)[None, :]).astype(np.float16)
    return x, W


def test_search_picks_the_constructed_optimum():
    P = lib()
    x, W = _known_optimum_case()
    err, best, alphas = P.awq_search_alpha(dev(x), dev(W))
    e = host(err)
    assert int(host(best)[0]) == 10 and alphas[10] == 0.5
    ref = O.search_errors(x, W, O.alpha_grid(20))
    # only the fp16 rounding of the layer output separates the two at alpha = 0.5
    y_ref = x.astype(np.float64) @ W.astype(np.float64).T
    assert e[10] <= np.sum((y_ref * 2.0 ** -11) ** 2)
    others = np.delete(np.arange(20), 10)
    assert np.all(np.abs(e[others] - ref[others]) <= 1e-2 * ref[others] + 1e-3 * e[10] + 1e-30)


@pytest.mark.parametrize("M,N,K", [(4, 64, 512), (48, 200, 1280), (1, 512, 512)])
def test_search_errors_match_the_oracle(M, N, K):
    P = lib()
    x, W = workloads.random_case(91 + M, M, N, K)
    err, best, _ = P.awq_search_alpha(dev(x), dev(W))
    e = host(err)
    ref = O.search_errors(x, W, O.alpha_grid(20))
    y_ref = x.astype(np.float64) @ W.astype(np.float64).T
    slack = 4 * np.sqrt(np.sum((y_ref * 2.0 ** -11) ** 2) * ref) + np.sum((y_ref * 2.0 ** -11) ** 2)
    assert np.all(np.abs(e - ref) <= 1e-3 * ref + slack), (e, ref)
    b = int(host(best)[0])
    assert e[b] == e.min() and b == int(np.argmin(e))
    order = np.sort(ref)
    if order[1] - order[0] > 2 * (1e-3 * order[1] + slack.max()):
        assert b == int(np.argmin(ref))


def test_search_reproducible():
    P = lib()
    x, W = workloads.random_case(97, 16, 256, 1024)
    e1 = host(P.awq_search_alpha(dev(x), dev(W))[0])
    e2 = host(P.awq_search_alpha(dev(x), dev(W))[0])
    assert np.array_equal(e1, e2)
