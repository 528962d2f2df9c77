"""Seeded synthetic inputs for the AWQ W4A16 g128 path.

This module only draws random numbers. It holds none of the method's
arithmetic: no scale, no fold, no quantization, no matmul. Both sides of
every parity test (the CPU oracle and the CUDA library) and ``bench.py``
take their inputs from here, so the two sides always see the same bytes.

Recipe (the pages name no dataset; these stand in for calibration text
and trained weights):

* activations ``x`` [M, K]: standard normal, drawn in fp32, with
  ``round(0.01 * K)`` input channels (the same channels for every row)
  multiplied by 20, then rounded to fp16 (round to nearest even).
  The outlier channels play the part of the ~1% salient channels that the
  CSDN overview of AWQ ("02.02 AWQ") describes.
* weights ``W`` [N, K] (row-major, K contiguous, like ``nn.Linear.weight``):
  normal with standard deviation 0.02, drawn in fp32, rounded to fp16.
* streams: ``numpy.random.default_rng([seed, workload_id, layer_idx, tag, ...])``;
  the weight stream does not depend on M, so a layer keeps its weights across
  the M values of a workload; the outlier channels come from a stream of their
  own, so they are the same for every M.
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

import numpy as np

OUTLIER_FRACTION = 0.01
OUTLIER_GAIN = 20.0
WEIGHT_STD = 0.02

_TAG_W = 1
_TAG_OUTLIER_COLS = 2
_TAG_X = 3


@dataclasses.dataclass(frozen=True)
class Layer:
    """One linear layer: y[M, N] = x[M, K] . W[N, K]^T."""

    name: str
    K: int
    N: int


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named set of layer shapes and token counts."""

    workload_id: int
    name: str
    layers: Tuple[Layer, ...]
    Ms: Tuple[int, ...]
    seed: int = 0
    description: str = ""


LLAMA2_7B = (
    Layer("qkv_fused", 4096, 12288),
    Layer("o_proj", 4096, 4096),
    Layer("gate_up_fused", 4096, 22016),
    Layer("down_proj", 11008, 4096),
)
LLAMA3_8B = (
    Layer("qkv_gqa", 4096, 6144),
    Layer("o_proj", 4096, 4096),
    Layer("gate_up_fused", 4096, 28672),
    Layer("down_proj", 14336, 4096),
)
LLAMA2_70B = (
    Layer("gate_up_70b", 8192, 28672),
    Layer("down_70b", 28672, 8192),
)

WORKLOADS = {
    "tiny_512": Workload(1, "tiny_512", (Layer("tiny", 512, 512),), (1,),
                         description="single 512x512 layer, M=1"),
    "llama2_7b_decode_m1": Workload(2, "llama2_7b_decode_m1", LLAMA2_7B, (1,),
                                    description="Llama-2-7B decode GEMV set, M=1"),
    "llama2_7b_decode_batched": Workload(3, "llama2_7b_decode_batched", LLAMA2_7B,
                                         (4, 8, 16, 32),
                                         description="Llama-2-7B batched decode"),
    "llama3_8b_prefill": Workload(4, "llama3_8b_prefill", LLAMA3_8B, (512, 2048, 4096),
                                  description="Llama-3-8B prefill GEMM"),
    "llama2_70b_layers": Workload(5, "llama2_70b_layers", LLAMA2_70B, (1, 16, 512),
                                  description="Llama-2-70B MLP layers"),
}


def n_outlier_channels(K: int) -> int:
    """round(0.01 * K): 5, 41, 110, 143, 82, 287 for K = 512, 4096, 11008, 14336, 8192, 28672."""
    return int(round(OUTLIER_FRACTION * K))


def outlier_channels(seed: int, workload_id: int, layer_idx: int, K: int) -> np.ndarray:
    """Sorted indices of the input channels that carry the x20 outliers."""
    rng = np.random.default_rng([seed, workload_id, layer_idx, _TAG_OUTLIER_COLS])
    return np.sort(rng.permutation(K)[: n_outlier_channels(K)])


def make_weight(seed: int, workload_id: int, layer_idx: int, N: int, K: int) -> np.ndarray:
    """W[N, K] fp16 ~ N(0, 0.02^2)."""
    rng = np.random.default_rng([seed, workload_id, layer_idx, _TAG_W])
    w = rng.standard_normal((N, K), dtype=np.float32)
    w *= np.float32(WEIGHT_STD)
    return w.astype(np.float16)


def make_activations(seed: int, workload_id: int, layer_idx: int, M: int, K: int) -> np.ndarray:
    """x[M, K] fp16 ~ N(0, 1) with round(0.01 K) channels scaled by 20."""
    rng = np.random.default_rng([seed, workload_id, layer_idx, _TAG_X, M])
    x = rng.standard_normal((M, K), dtype=np.float32)
    cols = outlier_channels(seed, workload_id, layer_idx, K)
    x[:, cols] *= np.float32(OUTLIER_GAIN)
    return x.astype(np.float16)


def layer_inputs(workload: Workload, layer_idx: int, M: int) -> Tuple[np.ndarray, np.ndarray]:
    """(x, W) for one layer of a workload at token count M."""
    layer = workload.layers[layer_idx]
    x = make_activations(workload.seed, workload.workload_id, layer_idx, M, layer.K)
    W = make_weight(workload.seed, workload.workload_id, layer_idx, layer.N, layer.K)
    return x, W


def random_case(seed: int, M: int, N: int, K: int) -> Tuple[np.ndarray, np.ndarray]:
    """(x, W) with the same recipe for an arbitrary test shape (workload id 99)."""
    x = make_activations(seed, 99, N * 7 + K, M, K)
    W = make_weight(seed, 99, N * 7 + K, N, K)
    return x, W


def workload_names() -> List[str]:
    return list(WORKLOADS)
