"""SVDQuant-style W4A4 + low-rank linear layer in fp64 (oracle; test infrastructure only).

What the layer computes ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", section
"SVDQuant deep dive"): weights and activations of the main transformer linears are both 4-bit
(W4A4); outliers are absorbed by a 16-bit low-rank branch, W = L1.L2 + R with only the residual R
quantized; the branch's down-projection X.L1 is fused with activation quantization and its
up-projection with the 4-bit GEMM. Quantization is post-training. The fused QKV and SwiGLU
epilogues follow the fused NVFP4 GEMMs of "FLUX 3 Image Klein on NVIDIA Blackwell", method 1.

Readings where the pages are silent (every one is listed in the design notes):
  * smoothing: lambda_j = sqrt(max_m |X_mj| / max_n |W_math[j, n]|) (migration strength 1/2), with
    lambda_j = 1 when either maximum is 0; inv_lambda = fp32(1 / lambda) and the exact-in-fp64
    lambda' = 1 / inv_lambda is what W is scaled by, so X.W = (X * inv_lambda).(lambda' * W)
    holds exactly in real arithmetic;
  * split: top-r truncated SVD of W_hat = diag(lambda').W_math with sigma folded into L1;
    L1s = bf16(diag(lambda')^-1 L1) (so the branch reads raw X), L2 = bf16(V_r^T), and
    R = fp32(W_hat - diag(lambda') L1s L2) absorbs the bf16 rounding of the branch;
  * calibration X is the layer's own X (no dataset): static activation scale = dynamic one;
  * SwiGLU: gate = columns [0, N/2), up = [N/2, N), bias added before silu,
    silu(z) = z / (1 + exp(-z)).
Shapes: X [M, K] (tokens x in-features), W [N, K] (nn.Linear layout), W_math = W.T [K, N].
"""
from __future__ import annotations

import numpy as np

from . import nvfp4
from .nvfp4 import f32


def bf16_round(x) -> np.ndarray:
    """Round fp64 values to bf16 (8 significant bits, round-half-even), returned as fp64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    out = np.ldexp(np.rint(m * 256.0), e - 8)
    nz = out != 0
    if (np.abs(out[nz]) < 2.0 ** -126).any() or (np.abs(out) > 3.3e38).any():
        raise ValueError("value outside bf16's normal range")
    return out


def smoothing(X: np.ndarray, W: np.ndarray):
    """Per-input-channel smoothing. X [M, K], W [N, K] (fp64 values of bf16 data).

    Returns (inv_lambda as fp32-valued fp64 [K], lambda' fp64 [K]).
    """
    a = np.abs(X).max(axis=0)
    b = np.abs(W).max(axis=0)
    ok = (a > 0) & (b > 0)
    lam = np.ones_like(a)
    lam[ok] = np.sqrt(a[ok] / b[ok])
    inv_lambda = f32(1.0 / lam)
    return inv_lambda, 1.0 / inv_lambda


def svd_split(W_hat: np.ndarray, r: int, lam_prime: np.ndarray):
    """Low-rank + residual split of W_hat [K, N]. Returns (L1s [K, r], L2 [r, N], R [K, N] fp32 values,
    sigma (all singular values of W_hat))."""
    K, N = W_hat.shape
    U, S, Vt = np.linalg.svd(W_hat, full_matrices=False)
    if r == 0:
        return np.zeros((K, 0)), np.zeros((0, N)), f32(W_hat), S
    L1 = U[:, :r] * S[:r]
    L1s = bf16_round(L1 / lam_prime[:, None])
    L2 = bf16_round(Vt[:r, :])
    R = f32(W_hat - (lam_prime[:, None] * L1s) @ L2)
    return L1s, L2, R, S


def prepare_layer(X: np.ndarray, W: np.ndarray, r: int) -> dict:
    """Offline (post-training) preparation of one layer from calibration X and weight W [N, K]."""
    inv_lambda, lam_prime = smoothing(X, W)
    W_hat = lam_prime[:, None] * W.T
    L1s, L2, R_kn, sigma = svd_split(W_hat, r, lam_prime)
    return {"inv_lambda": inv_lambda, "lam_prime": lam_prime, "L1s": L1s, "L2": L2,
            "R": np.ascontiguousarray(R_kn.T), "sigma": sigma, "r": r}


def add_lora(prep: dict, A: np.ndarray, B: np.ndarray) -> dict:
    """The layer with a LoRA adapter (A [K, r_l], B [r_l, N], bf16 values) riding on the 16-bit
    branch: L1s <- [L1s | A], L2 <- [L2 ; B], rank r + r_l. The pages only name LoRA support
    ("Bringing Nunchaku 4-bit diffusion inference to Diffusers"); the concatenation is a reading:
    the branch reads raw X, as a LoRA adapter does, so (X [L1s|A]) [L2;B] = X L1s L2 + X A B."""
    out = dict(prep)
    K = prep["inv_lambda"].shape[0]
    L1s = prep["L1s"] if prep["r"] > 0 else np.zeros((K, 0))
    L2 = prep["L2"] if prep["r"] > 0 else np.zeros((0, B.shape[1]))
    out["L1s"] = np.concatenate([L1s, np.asarray(A, dtype=np.float64)], axis=1)
    out["L2"] = np.concatenate([L2, np.asarray(B, dtype=np.float64)], axis=0)
    out["r"] = prep["r"] + A.shape[1]
    return out


def smooth_activations(X: np.ndarray, inv_lambda: np.ndarray) -> np.ndarray:
    """x_hat = fp32(x * inv_lambda_k); one rounding (bf16 x fp32 is exact in fp64)."""
    return f32(X * inv_lambda[None, :])


def calibrate_activation_scale(X: np.ndarray, inv_lambda: np.ndarray) -> float:
    return nvfp4.tensor_scale(np.abs(smooth_activations(X, inv_lambda)).max())


def quantize_activations(X: np.ndarray, inv_lambda: np.ndarray, g_x: float):
    return nvfp4.quantize(smooth_activations(X, inv_lambda), g_x)


def quantize_weight(R: np.ndarray):
    """R [N, K] fp32 values -> (g_w, codes [N, K], scales [N, K/16])."""
    g_w = nvfp4.tensor_scale(np.abs(R).max())
    codes, scales = nvfp4.quantize(R, g_w)
    return g_w, codes, scales


def silu(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def apply_swiglu(y: np.ndarray) -> np.ndarray:
    half = y.shape[-1] // 2
    return silu(y[..., :half]) * y[..., half:]


def layer_forward(X, prep, g_x, weight_q, bias=None, swiglu=False) -> np.ndarray:
    """y = g_x g_w (Xq . Rq^T) + (X L1s) L2 + bias, then SwiGLU if asked; fp64 [M, N or N/2]."""
    g_w, wc, ws = weight_q
    xc, xs = quantize_activations(X, prep["inv_lambda"], g_x)
    acc = nvfp4.block_values(xc, xs) @ nvfp4.block_values(wc, ws).T
    y = (g_x * g_w) * acc
    if prep["r"] > 0:
        y = y + (X @ prep["L1s"]) @ prep["L2"]
    if bias is not None:
        y = y + bias[None, :]
    return apply_swiglu(y) if swiglu else y


def layer_outputs_at(X, prep, g_x, weight_q, rows, cols, bias=None, swiglu=False) -> np.ndarray:
    """The same y as ``layer_forward`` but only at (rows[i], cols[i]), one output at a time."""
    g_w, wc, ws = weight_q
    N = wc.shape[0]
    out = np.empty(len(rows))
    xrow_cache = {}
    for i, (m, n) in enumerate(zip(rows, cols)):
        if m not in xrow_cache:
            xc, xs = quantize_activations(X[m:m + 1], prep["inv_lambda"], g_x)
            u = X[m] @ prep["L1s"] if prep["r"] > 0 else None
            xrow_cache[m] = (nvfp4.block_values(xc, xs)[0], u)
        xv, u = xrow_cache[m]

        def one(col):
            wv = nvfp4.block_values(wc[col:col + 1], ws[col:col + 1])[0]
            v = (g_x * g_w) * float(xv @ wv)
            if u is not None:
                v += float(u @ prep["L2"][:, col])
            if bias is not None:
                v += bias[col]
            return v

        if swiglu:
            out[i] = float(silu(np.float64(one(n))) * one(N // 2 + n))
        else:
            out[i] = one(n)
    return out
