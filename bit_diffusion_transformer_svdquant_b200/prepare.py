"""Offline (post-training) preparation of one layer's weight for svdq_pack_weight.

Post-training quantization ("Bringing Nunchaku 4-bit diffusion inference to Diffusers", "SVDQuant
deep dive") splits each weight once, offline: smoothing factors from calibration activations, a
top-r SVD of the smoothed weight for the 16-bit branch, and the residual that gets quantized. This
step sits before the C ABI (whose first call, svdq_pack_weight, takes the residual) and is not on the
per-step path; it uses torch's fp64 linear algebra (the SVD is a library routine).

Readings (the pages give no formula): lambda_j = sqrt(max|X_j| / max|W_j|) per input channel
(1 where either is 0); L1s = bf16(diag(lambda)^-1 U_r S_r), L2 = bf16(V_r^T);
R = fp32(W_hat - diag(lambda) L1s L2), so that the bf16 rounding of the branch is absorbed by R.
"""
from __future__ import annotations

import torch


@torch.no_grad()
def prepare_layer(X: torch.Tensor, W: torch.Tensor, r: int, device=None) -> dict:
    """X [M, K] bf16 calibration activations, W [N, K] bf16 weight -> dict of R [N, K] fp32,
    L1s [K, r] bf16, L2 [r, N] bf16, inv_lambda [K] fp32, all on ``device``."""
    device = X.device if device is None else device
    Xd = X.to(device=device, dtype=torch.float64)
    Wd = W.to(device=device, dtype=torch.float64)
    a = Xd.abs().amax(dim=0)
    b = Wd.abs().amax(dim=0)
    ok = (a > 0) & (b > 0)
    lam = torch.where(ok, torch.sqrt(a / torch.where(ok, b, torch.ones_like(b))), torch.ones_like(a))
    inv_lambda = (1.0 / lam).to(torch.float32)
    lam_p = 1.0 / inv_lambda.to(torch.float64)
    W_hat = lam_p[:, None] * Wd.T
    N = W.shape[0]
    if r == 0:
        R = W_hat.to(torch.float32).T.contiguous()
        return {"R": R, "L1s": None, "L2": None, "inv_lambda": inv_lambda.contiguous()}
    U, S, Vh = torch.linalg.svd(W_hat, full_matrices=False)
    L1s = (U[:, :r] * S[:r] / lam_p[:, None]).to(torch.float32).to(torch.bfloat16)
    L2 = Vh[:r].to(torch.float32).to(torch.bfloat16)
    R = (W_hat - (lam_p[:, None] * L1s.to(torch.float64)) @ L2.to(torch.float64)).to(torch.float32)
    del U, S, Vh, W_hat
    return {"R": R.T.contiguous(), "L1s": L1s.contiguous(), "L2": L2.contiguous(),
            "inv_lambda": inv_lambda.contiguous(), "N": N}


@torch.no_grad()
def concat_lora(prep: dict, A: torch.Tensor, B: torch.Tensor) -> dict:
    """A LoRA adapter (A [K, r_l], B [r_l, N]) rides on the 16-bit branch: L1s <- [L1s | A],
    L2 <- [L2 ; B] in bf16, so the packed layer computes X L1s L2 + X A B with the same kernels.
    The pages only name LoRA support; the concatenation is a reading (the branch reads raw X, as a
    LoRA adapter does). The total rank must be one the kernels take (16, 32 or 64)."""
    r0 = 0 if prep["L1s"] is None else prep["L1s"].shape[1]
    r = r0 + A.shape[1]
    if r not in (16, 32, 64):
        raise ValueError(f"rank {r0} + LoRA {A.shape[1]} = {r} is not one of 16, 32, 64")
    dev = prep["inv_lambda"].device
    A = A.to(device=dev, dtype=torch.bfloat16)
    B = B.to(device=dev, dtype=torch.bfloat16)
    out = dict(prep)
    out["L1s"] = A.contiguous() if r0 == 0 else torch.cat([prep["L1s"], A], dim=1).contiguous()
    out["L2"] = B.contiguous() if r0 == 0 else torch.cat([prep["L2"], B], dim=0).contiguous()
    return out
