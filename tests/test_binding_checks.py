"""The Python binding's argument checks, on CPU tensors (no device call is made).

Every public call validates its tensors before it reaches the C ABI: a buffer
too small for the packed layout, a scale vector of the wrong length or an
output of the wrong shape would otherwise become out-of-bounds copies on the
GPU. The validators take ``require_cuda=False`` here so that the size logic
runs without a device; the public calls always require CUDA tensors on the
current device.
"""
import pytest
import torch

import weight_only_quantization_w4a16_b200 as P
from oracle import awq_oracle as O


def _packed(N, K, shrink=None):
    qb, sb, zb = P._packed_sizes_host(N, K)
    q = torch.empty(qb // 4 - (1 if shrink == "q" else 0), dtype=torch.int32)
    s = torch.empty(sb // 2 - (1 if shrink == "s" else 0), dtype=torch.float16)
    z = torch.empty(zb - (1 if shrink == "z" else 0), dtype=torch.uint8)
    return q, s, z


@pytest.mark.parametrize("N,K", [(1, 128), (300, 256), (7, 1152), (4096, 11008)])
def test_host_sizes_agree_with_the_oracle_layout(N, K):
    words, halves, zbytes = O.packed_sizes(N, K)
    assert P._packed_sizes_host(N, K) == (4 * words, 2 * halves, zbytes)


def test_quantize_rejects_short_outputs_and_wrong_fold_length():
    W = torch.zeros((300, 256), dtype=torch.float16)
    P.validate_quantize(W, torch.ones(256), _packed(300, 256), require_cuda=False)
    for which in ("q", "s", "z"):
        with pytest.raises(ValueError, match="too small"):
            P.validate_quantize(W, None, _packed(300, 256, shrink=which), require_cuda=False)
    with pytest.raises(ValueError, match="K=256"):
        P.validate_quantize(W, torch.ones(255), _packed(300, 256), require_cuda=False)
    with pytest.raises(ValueError, match="multiple of 128"):
        P.validate_quantize(torch.zeros((8, 200), dtype=torch.float16), None, _packed(8, 256), require_cuda=False)


def test_linear_rejects_wrong_y_shape_and_short_weights():
    x = torch.zeros((3, 512), dtype=torch.float16)
    P.validate_linear(x, *_packed(64, 512), 64, torch.empty((3, 64), dtype=torch.float16), require_cuda=False)
    with pytest.raises(ValueError, match="shape"):
        P.validate_linear(x, *_packed(64, 512), 64, torch.empty((3, 65), dtype=torch.float16), require_cuda=False)
    with pytest.raises(ValueError, match="too small"):
        P.validate_linear(x, *_packed(64, 512, shrink="q"), 64, torch.empty((3, 64), dtype=torch.float16),
                          require_cuda=False)
    # packed for a smaller K than x has
    with pytest.raises(ValueError, match="too small"):
        P.validate_linear(x, *_packed(64, 256), 64, torch.empty((3, 64), dtype=torch.float16), require_cuda=False)


def test_activation_checks():
    x = torch.zeros((4, 256), dtype=torch.float16)
    P.validate_activation_scale(x, torch.empty(256), torch.empty((4, 256), dtype=torch.float16), require_cuda=False)
    P.validate_activation_scale(x, torch.empty(256), None, require_cuda=False)
    with pytest.raises(ValueError, match="K=256"):
        P.validate_activation_scale(x, torch.empty(128), None, require_cuda=False)
    with pytest.raises(ValueError, match="shape"):
        P.validate_activation_scale(x, torch.empty(256), torch.empty((2, 256), dtype=torch.float16),
                                    require_cuda=False)
    with pytest.raises(ValueError, match="K=256"):
        P.validate_scale_activations(x, torch.empty(255), torch.empty((4, 256), dtype=torch.float16),
                                     require_cuda=False)
    with pytest.raises(ValueError, match="shape"):
        P.validate_scale_activations(x, torch.empty(256), torch.empty((4, 128), dtype=torch.float16),
                                     require_cuda=False)


def test_dtype_and_cuda_requirements():
    W = torch.zeros((16, 128), dtype=torch.float32)
    with pytest.raises(TypeError, match="float16"):
        P.validate_quantize(W, None, _packed(16, 128), require_cuda=False)
    with pytest.raises(ValueError, match="CUDA"):
        P.validate_quantize(W.half(), None, _packed(16, 128))
