"""Seeded synthetic inputs for the W4A4 + low-rank linear layer.

This module is the one piece of code that the CUDA path and the CPU oracle share. It draws random
numbers and rounds the draws to bf16, the layer's input dtype; it holds none of the quantization
method's arithmetic (no smoothing, no SVD, no NVFP4 rounding).

Workloads follow the token counts of a FLUX-class diffusion transformer: every latent token is one
16x16-pixel patch, so a 1024x1024 image is a 64x64 = 4096-token grid and a 2048x2048 image a
128x128 = 16384-token grid; a reference image adds its own grid of tokens (FLUX.3 Klein in Diffusers,
"How it works" section; FLUX.3 Klein open-weights article, reference-image timing). 512 text tokens
are added to every image workload. Hidden size 3072, MLP width 12288 and rank 32 are the layer
shapes the workload table fixes; the pages give no parameter count.

Draw recipe for one linear layer (numpy PCG64, ``default_rng([seed, layer])``):
  1. X ~ N(0, 1) in fp64, shape [M, K];
  2. ``n_out = round(p * K)`` outlier channels chosen without replacement;
  3. those whole columns of X multiplied by the outlier scale (x40 or x50);
  4. X rounded to bf16 (round-to-nearest-even through fp32, torch's conversion);
  5. W ~ N(0, 1/K) read as a variance (std K**-0.5), drawn in nn.Linear layout [N, K], then bf16;
  6. bias ~ N(0, 0.02) read as a variance (std 0.02**0.5), then bf16 (only where the workload
     has a bias).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class LinearSpec:
    """One W4A4 + low-rank linear layer: y = X @ W.T (+ bias) with an optional SwiGLU."""
    name: str
    M: int
    K: int
    N: int
    r: int
    outlier_frac: float
    outlier_scale: float
    bias: bool
    swiglu: bool = False
    layer: int = 0


@dataclass(frozen=True)
class Workload:
    name: str
    description: str
    layers: tuple = field(default_factory=tuple)


def _qkv(name, M, layer=0, bias=True):
    return LinearSpec(name, M, 3072, 9216, 32, 0.01, 50.0, bias, False, layer)


WORKLOADS = {
    "tiny": Workload(
        "tiny", "tiny W4A4 linear 256x512x512, r=16, 2% outlier channels x40, no bias",
        (LinearSpec("tiny", 256, 512, 512, 16, 0.02, 40.0, False),)),
    "qkv_1024": Workload(
        "qkv_1024", "1024^2 text-to-image fused QKV: M=4608 (4096 image + 512 text), K=3072, N=9216, r=32, bias",
        (_qkv("qkv_1024", 4608),)),
    "mlp_1024": Workload(
        "mlp_1024", "1024^2 SwiGLU MLP: gate/up 4608x3072 -> 2x12288 with SwiGLU, down 4608x12288 -> 3072, r=32",
        (LinearSpec("mlp_1024.gate_up", 4608, 3072, 24576, 32, 0.01, 50.0, True, True, 0),
         LinearSpec("mlp_1024.down", 4608, 12288, 3072, 32, 0.01, 50.0, True, False, 1))),
    "qkv_2048": Workload(
        "qkv_2048", "2048^2 generation fused QKV: M=16896 (16384 image + 512 text), K=3072, N=9216, r=32, no bias",
        (_qkv("qkv_2048", 16896, bias=False),)),
    "edit_2048": Workload(
        "edit_2048", "2048^2 edit with one 2048^2 reference: M=33280, QKV 3072->9216 then out-proj 3072->3072, r=32",
        (_qkv("edit_2048.qkv", 33280, 0),
         LinearSpec("edit_2048.out", 33280, 3072, 3072, 32, 0.01, 50.0, True, False, 1))),
}


def _to_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_linear_inputs(spec: LinearSpec, seed: int = 0, M: int | None = None) -> dict:
    """Draw X, W (and bias) for ``spec`` on the CPU. ``M`` overrides the token count (row subset
    draws: the first M rows of the full draw are NOT reproduced, use the full M for parity)."""
    M = spec.M if M is None else M
    rng = np.random.default_rng([seed, spec.layer])
    X = rng.standard_normal((M, spec.K))
    n_out = int(round(spec.outlier_frac * spec.K))
    channels = np.sort(rng.choice(spec.K, size=n_out, replace=False))
    X[:, channels] *= spec.outlier_scale
    W = rng.standard_normal((spec.N, spec.K)) * (1.0 / np.sqrt(spec.K))
    out = {"X": _to_bf16(X), "W": _to_bf16(W), "outlier_channels": channels}
    if spec.bias:
        out["bias"] = _to_bf16(rng.standard_normal(spec.N) * np.sqrt(0.02))
    return out


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw uint16 bit patterns of a bf16 tensor (for byte-level handoff)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_values(t: torch.Tensor) -> np.ndarray:
    """The exact values of a bf16 tensor as fp64."""
    return t.to(torch.float64).numpy()
