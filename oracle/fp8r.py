"""Row-wise FP8 (W8A8) variant of the layer (oracle; test infrastructure only, see ``oracle/__init__``).

The pages name a second quantized format next to NVFP4: FP8 with one scale per row ("FLUX 3
Image Klein on NVIDIA Blackwell", "Method 1: quantization (NVFP4 / FP8)"; the Diffusers release
notes for FLUX.3 Image Klein list NVFP4 and row-wise FP8 "fp8r" single-file weights, with fast
kernels from compute capability 8.9 on). They give no formula; the readings taken here are:

  * the layer keeps its SVDQuant structure (smoothing, 16-bit low-rank branch, quantized residual
    R); only the 4-bit operands become E4M3 with one fp32 scale per row: per output row of R and
    per token row of the smoothed activations (computed from the call's own X);
  * row scale s = fp32(amax_row / 448); a row whose amax is below 2**-100 (zero included) gets
    s = 1; codes q = E4M3(fp32(v * fp32(1 / s))), round to nearest, ties to the even code,
    saturating at 448, the sign kept when the magnitude rounds to 0 (as for NVFP4);
  * decoded element: dec(q) * s; the main product is s_x[m] * s_w[n] * sum_k dec(qx) dec(qw),
    then the branch (X L1s) L2, the bias and SwiGLU exactly as in the NVFP4 layer.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4
from .nvfp4 import f32
from .svdquant import apply_swiglu, smooth_activations

ROW_MAX = nvfp4.E4M3_MAX  # 448


def row_scales(v32: np.ndarray) -> np.ndarray:
    """fp32 scale per row: fp32(amax / 448), 1 for rows whose amax is below 2**-100."""
    amax = np.abs(np.asarray(v32, dtype=np.float64)).max(axis=1)
    s = f32(amax / ROW_MAX)
    return np.where(amax < nvfp4.TINY_AMAX, 1.0, s)


def quantize_rows(v32: np.ndarray):
    """fp32 values [rows, K] -> (scales fp32 [rows], E4M3 codes uint8 [rows, K])."""
    v = np.asarray(v32, dtype=np.float64)
    s = row_scales(v)
    rs = f32(1.0 / s)
    codes = nvfp4.e4m3_encode(f32(v * rs[:, None]))
    return s, codes


def dequantize_rows(scales: np.ndarray, codes: np.ndarray) -> np.ndarray:
    return nvfp4.e4m3_decode(codes) * np.asarray(scales, dtype=np.float64)[:, None]


def quantize_weight(R: np.ndarray):
    """R [N, K] fp32 values -> (row scales [N], codes [N, K])."""
    return quantize_rows(R)


def quantize_activations(X: np.ndarray, inv_lambda: np.ndarray):
    """Smoothed activations, one scale per token row (dynamic: from this X)."""
    return quantize_rows(smooth_activations(X, inv_lambda))


def layer_forward(X, prep, weight_q, bias=None, swiglu=False) -> np.ndarray:
    """y = s_x s_w (Xq . Rq^T) + (X L1s) L2 + bias, then SwiGLU if asked; fp64 [M, N or N/2]."""
    sw, qw = weight_q
    sx, qx = quantize_activations(X, prep["inv_lambda"])
    acc = nvfp4.e4m3_decode(qx) @ nvfp4.e4m3_decode(qw).T
    y = sx[:, None] * sw[None, :] * acc
    if prep["r"] > 0:
        y = y + (X @ prep["L1s"]) @ prep["L2"]
    if bias is not None:
        y = y + bias[None, :]
    return apply_swiglu(y) if swiglu else y
