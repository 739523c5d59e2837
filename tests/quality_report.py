"""Informational quality of the quantized layer (reported, not a parity gate; oracle only).

For each layer of a workload, the relative Frobenius error ||y - y_exact|| / ||y_exact|| of the
oracle's layer output against the unquantized fp64 product y_exact = X W^T (+ bias), for

  plain W4A4    no smoothing, no low-rank branch
  smoothing     smoothing, no branch
  branch        no smoothing, rank-r branch
  SVDQuant      smoothing + rank-r branch (what the library computes)
  FP8 row-wise  smoothing + rank-r branch, E4M3 codes with one scale per row

Smoothing factors and the static activation scale come from the layer's full X (the calibration
reading: the layer's own X); the error is measured on its first `rows` rows. Inputs are the seeded
synthetic workloads.

  python tests/quality_report.py [--rows 1024] [workload ...]
"""
from __future__ import annotations

import argparse
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_diffusion_transformer_svdquant_b200 import synth  # noqa: E402
from oracle import fp8r, svdquant  # noqa: E402


def _unsmoothed(W, r):
    """prepare_layer's split with lambda = 1 (no smoothing)."""
    K = W.shape[1]
    ones = np.ones(K)
    L1s, L2, R_kn, sigma = svdquant.svd_split(W.T, r, ones)
    return {"inv_lambda": ones, "lam_prime": ones, "L1s": L1s, "L2": L2, "R": np.ascontiguousarray(R_kn.T),
            "sigma": sigma, "r": r}


def layer_errors(X, W, b, r, rows):
    """Relative errors of the five variants on X[:rows] (calibrated on all of X)."""
    Xs = X[:rows]
    exact = Xs @ W.T + (0.0 if b is None else b[None, :])
    nrm = np.linalg.norm(exact)
    out = {}
    for name, smooth, rr in (("plain W4A4", False, 0), ("smoothing", True, 0), ("branch", False, r),
                             ("SVDQuant", True, r)):
        p = svdquant.prepare_layer(X, W, rr) if smooth else _unsmoothed(W, rr)
        g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
        y = svdquant.layer_forward(Xs, p, g_x, svdquant.quantize_weight(p["R"]), b)
        out[name] = float(np.linalg.norm(y - exact) / nrm)
        if name == "SVDQuant":
            y8 = fp8r.layer_forward(Xs, p, fp8r.quantize_weight(p["R"]), b)
            out["FP8 row-wise"] = float(np.linalg.norm(y8 - exact) / nrm)
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=1024)
    ap.add_argument("workloads", nargs="*", default=["tiny", "qkv_1024", "mlp_1024", "qkv_2048", "edit_2048"])
    args = ap.parse_args()
    cols = ["plain W4A4", "smoothing", "branch", "SVDQuant", "FP8 row-wise"]
    print("| layer (M×K×N, r) | " + " | ".join(cols) + " |")
    print("|---|" + "---|" * len(cols))
    for name in args.workloads:
        for spec in synth.WORKLOADS[name].layers:
            t0 = time.perf_counter()
            d = synth.make_linear_inputs(spec)
            X, W = synth.bf16_values(d["X"]), synth.bf16_values(d["W"])
            b = synth.bf16_values(d["bias"]) if spec.bias else None
            e = layer_errors(X, W, b, spec.r, min(args.rows, spec.M))
            print(f"| {name} {spec.M}×{spec.K}×{spec.N}, r={spec.r} | "
                  + " | ".join(f"{e[c]:.2e}" for c in cols) + f" |  <!-- {time.perf_counter() - t0:.0f} s -->",
                  flush=True)


if __name__ == "__main__":
    main()
