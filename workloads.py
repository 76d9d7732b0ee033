"""Seeded synthetic inputs for the SVDQuant W4A4 + low-rank linear layer.

This module only draws random tensors with the shapes and value distributions
of the FLUX-shaped workloads; it holds none of the method's arithmetic (no
smoothing factor, no SVD, no quantization).  Both the CPU oracle (tests) and
the CUDA path (tests, bench) take their inputs from here, so the two sides see
bit-identical bf16 data.

Recipe (same for every layer):
  * one ``torch.Generator('cpu')`` for the weight-side tensors, seeded with the
    layer's seed, drawing in order: W ~ N(0, w_std) (K x N), then the outlier
    input rows of W (``randperm``), then bias ~ N(0, 0.01), then the LoRA
    factors A (K x r_lora) and B (r_lora x N) ~ N(0, 0.01);
  * a second generator for the activations, seeded with ``seed + 7919``,
    drawing X ~ N(0, 1) (M x K) and then the outlier channels (``randperm``),
    whose columns are multiplied by 30;
  * everything is drawn in fp32 and rounded to bf16 (round to nearest even).

Diffusion-model checkpoints and prompt datasets are not available, so these
tensors stand in for the FLUX.1 linear layers the SVDQuant paper (arXiv
2411.05007, Sec. 5.1) quantizes; the shapes are those of FLUX.1 attention and
MLP projections at 4096 image + 512 text tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np
import torch

NVFP4 = "nvfp4"
INT4 = "int4"


@dataclass(frozen=True)
class LayerSpec:
    name: str
    K: int
    N: int
    rank: int = 32
    fmt: str = NVFP4
    bias: bool = False
    lora_rank: int = 0
    x_outliers: int = 8            # outlier input channels of X (x30)
    w_outlier_rows: int = 0        # outlier input rows of W (x10)
    w_std: float = 0.02
    seed: int = 0


@dataclass(frozen=True)
class ConfigSpec:
    name: str
    description: str
    layers: List[LayerSpec]
    Ms: List[int] = field(default_factory=list)


def _c1_outliers(K: int) -> int:
    """8 outlier channels per 1024 input channels (the 256x1024 layer's ratio)."""
    return max(1, (8 * K) // 1024)


CONFIGS: Dict[str, ConfigSpec] = {
    "c1_small": ConfigSpec(
        "c1_small", "single NVFP4 layer 256x1024->1024, r=32",
        [LayerSpec("linear", 1024, 1024, x_outliers=8, seed=0)], [256]),
    "c2_qkv": ConfigSpec(
        "c2_qkv", "FLUX attention QKV 4608x3072->9216, NVFP4, r=32",
        [LayerSpec("qkv", 3072, 9216, x_outliers=30, w_outlier_rows=15, seed=0)], [4608]),
    "c3_mlp": ConfigSpec(
        "c3_mlp", "FLUX MLP pair fc1 3072->12288, fc2 12288->3072, NVFP4, r=32, bias",
        [LayerSpec("fc1", 3072, 12288, bias=True, x_outliers=_c1_outliers(3072), seed=0),
         LayerSpec("fc2", 12288, 3072, bias=True, x_outliers=_c1_outliers(12288), seed=1)],
        [4608]),
    "c4_int4_lora": ConfigSpec(
        "c4_int4_lora", "INT4 g64 4608x3072->3072, r=32 + LoRA 16 folded into r=48",
        [LayerSpec("proj", 3072, 3072, fmt=INT4, lora_rank=16,
                   x_outliers=_c1_outliers(3072), seed=0)], [4608]),
    "c5_block": ConfigSpec(
        "c5_block", "DiT block qkv/out/fc1/fc2 at M = 1024, 4096, 16384, NVFP4, r=32, bias",
        [LayerSpec("qkv", 3072, 9216, bias=True, x_outliers=_c1_outliers(3072), seed=0),
         LayerSpec("out", 3072, 3072, bias=True, x_outliers=_c1_outliers(3072), seed=1),
         LayerSpec("fc1", 3072, 12288, bias=True, x_outliers=_c1_outliers(3072), seed=2),
         LayerSpec("fc2", 12288, 3072, bias=True, x_outliers=_c1_outliers(12288), seed=3)],
        [1024, 4096, 16384]),
}


def layer_spec(config: str, layer: Optional[str] = None) -> LayerSpec:
    cfg = CONFIGS[config]
    if layer is None:
        return cfg.layers[0]
    for spec in cfg.layers:
        if spec.name == layer:
            return spec
    raise KeyError(f"{config} has no layer {layer}")


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a bf16 tensor as a uint16 numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def make_weights(spec: LayerSpec, K: Optional[int] = None, N: Optional[int] = None):
    """W (K x N), bias (N) and LoRA A/B as bf16 CPU tensors (None where absent)."""
    K = spec.K if K is None else K
    N = spec.N if N is None else N
    g = torch.Generator().manual_seed(spec.seed)
    W = torch.randn(K, N, generator=g) * spec.w_std
    if spec.w_outlier_rows:
        n_rows = max(1, (spec.w_outlier_rows * K) // spec.K)
        rows = torch.randperm(K, generator=g)[:n_rows]
        W[rows] *= 10.0
    bias = (torch.randn(N, generator=g) * 0.01).to(torch.bfloat16) if spec.bias else None
    A = B = None
    if spec.lora_rank:
        A = (torch.randn(K, spec.lora_rank, generator=g) * 0.01).to(torch.bfloat16)
        B = (torch.randn(spec.lora_rank, N, generator=g) * 0.01).to(torch.bfloat16)
    return W.to(torch.bfloat16), bias, A, B


def make_activations(spec: LayerSpec, M: int, K: Optional[int] = None) -> torch.Tensor:
    """X (M x K) as a bf16 CPU tensor: N(0,1) with outlier channels x30."""
    K = spec.K if K is None else K
    g = torch.Generator().manual_seed(spec.seed + 7919)
    X = torch.randn(M, K, generator=g)
    n_out = max(1, (spec.x_outliers * K) // spec.K)
    cols = torch.randperm(K, generator=g)[:n_out]
    X[:, cols] *= 30.0
    return X.to(torch.bfloat16)


def make_layer(config: str, layer: Optional[str] = None, M: Optional[int] = None):
    """All inputs of one layer of a named workload at its (first) token count."""
    spec = layer_spec(config, layer)
    if M is None:
        M = CONFIGS[config].Ms[0]
    W, bias, A, B = make_weights(spec)
    X = make_activations(spec, M)
    return {"spec": spec, "M": M, "X": X, "W": W, "bias": bias, "lora_A": A, "lora_B": B}


def make_small(M: int, K: int, N: int, rank: int = 32, fmt: str = NVFP4, seed: int = 0,
               bias: bool = False, lora_rank: int = 0, x_outliers: int = 8,
               w_outlier_rows: int = 0):
    """A small layer with the config-1 distributions at arbitrary sizes."""
    spec = LayerSpec("small", K, N, rank=rank, fmt=fmt, bias=bias, lora_rank=lora_rank,
                     x_outliers=min(x_outliers, K), w_outlier_rows=w_outlier_rows, seed=seed)
    W, b, A, B = make_weights(spec)
    X = make_activations(spec, M)
    return {"spec": spec, "M": M, "X": X, "W": W, "bias": b, "lora_A": A, "lora_B": B}
