"""Shared helpers for the GPU parity tests: run the oracle and the CUDA path on the same inputs and
compare. Inputs come from the seeded generator or are built by hand; expected values come only
from ``oracle/``."""
from __future__ import annotations

import numpy as np
import torch

import bit_diffusion_transformer_svdquant_b200 as svdq
from oracle import nvfp4, svdquant

REL_TOL = 2e-3   # max|y - y_ref| <= REL_TOL * max|y_ref|, fp32-output mode


def to_dev_bf16(a: np.ndarray, dev) -> torch.Tensor:
    """fp64 array of bf16-representable values -> exact bf16 device tensor."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), a), "value not representable in bf16"
    return t.to(dev)


def to_dev_f32(a: np.ndarray, dev) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(dev)


def oracle_act_codes(X, inv_lambda, g_x, chunk=4096):
    """Oracle activation codes (packed nibbles) and scales, row chunk by row chunk."""
    M, K = X.shape
    codes = np.empty((M, K // 2), np.uint8)
    scales = np.empty((M, K // 16), np.uint8)
    for i in range(0, M, chunk):
        q, s = svdquant.quantize_activations(X[i:i + chunk], inv_lambda, g_x)
        codes[i:i + chunk] = nvfp4.pack_nibbles(q)
        scales[i:i + chunk] = s
    return codes, scales


class Case:
    """One layer run through both the oracle and the library."""

    def __init__(self, X, W, bias, r, swiglu, dev, prep=None, g_x=None):
        self.X, self.W, self.bias, self.r, self.swiglu, self.dev = X, W, bias, r, swiglu, dev
        self.prep = svdquant.prepare_layer(X, W, r) if prep is None else prep
        p = self.prep
        self.g_x_ref = svdquant.calibrate_activation_scale(X, p["inv_lambda"]) if g_x is None else g_x
        self.wq = svdquant.quantize_weight(p["R"])
        self.Xd = to_dev_bf16(X, dev)
        self.bias_d = None if bias is None else to_dev_bf16(bias, dev)
        self.w = svdq.PackedWeight(to_dev_f32(p["R"], dev),
                                   to_dev_bf16(p["L1s"], dev) if r else None,
                                   to_dev_bf16(p["L2"], dev) if r else None,
                                   to_dev_f32(p["inv_lambda"], dev), swiglu=swiglu)
        if g_x is None:
            self.g_x = svdq.calibrate_act(self.Xd, self.w)
        else:
            self.g_x = torch.tensor([g_x], dtype=torch.float32, device=dev)
        self.act = svdq.QuantizedAct(X.shape[0], X.shape[1], r, dev)
        svdq.quantize_act(self.Xd, self.w, self.g_x, self.act)

    def run_gemm(self, out_dtype):
        return svdq.gemm(self.act, self.w, self.bias_d, out_dtype=out_dtype)

    # ---- checks
    def check_scales(self):
        assert float(self.g_x.item()) == self.g_x_ref, (self.g_x.item(), self.g_x_ref)
        assert float(self.w.g_w().item()) == self.wq[0], (self.w.g_w().item(), self.wq[0])
        alpha = float(np.float32(np.float32(self.g_x_ref) * np.float32(self.wq[0])))
        assert float(self.act.alpha().item()) == alpha

    def check_weight_codes(self):
        c, s = svdq.export_weight(self.w)
        c, s = c.cpu().numpy(), s.cpu().numpy()
        ref_c = nvfp4.pack_nibbles(self.wq[1])
        bad = np.nonzero((c != ref_c).any(axis=1))[0]
        assert bad.size == 0, f"weight code rows differ: {bad[:10]}"
        assert np.array_equal(s, self.wq[2]), f"weight scales differ at {np.argwhere(s != self.wq[2])[:10]}"

    def check_act_codes(self):
        c, s = svdq.export_act(self.act)
        c, s = c.cpu().numpy(), s.cpu().numpy()
        ref_c, ref_s = oracle_act_codes(self.X, self.prep["inv_lambda"], self.g_x_ref)
        if not np.array_equal(s, ref_s):
            raise AssertionError(f"act scales differ at {np.argwhere(s != ref_s)[:10]}")
        if not np.array_equal(c, ref_c):
            idx = np.argwhere(c != ref_c)[:10]
            raise AssertionError(f"act codes differ at {idx}: got {[hex(c[tuple(i)]) for i in idx]} "
                                 f"want {[hex(ref_c[tuple(i)]) for i in idx]}")

    def y_ref_full(self):
        return svdquant.layer_forward(self.X, self.prep, self.g_x_ref, self.wq, self.bias, self.swiglu)

    def y_ref_at(self, rows, cols):
        return svdquant.layer_outputs_at(self.X, self.prep, self.g_x_ref, self.wq, rows, cols, self.bias,
                                         self.swiglu)

    def check_outputs(self, samples=None, seed=0):
        y32 = self.run_gemm(torch.float32)
        ybf = self.run_gemm(torch.bfloat16)
        torch.cuda.synchronize()
        assert svdq.device_status() == 0
        # bf16 output is exactly the bf16 rounding of the fp32 output
        assert torch.equal(ybf, y32.to(torch.bfloat16))
        y = y32.cpu().numpy().astype(np.float64)
        assert np.isfinite(y).all()
        if samples is None:
            ref = self.y_ref_full()
            err = np.max(np.abs(y - ref))
            scale = np.max(np.abs(ref))
        else:
            M, Nout = y.shape
            rng = np.random.default_rng(seed)
            rows = np.concatenate([rng.integers(0, M, samples), [0, M - 1, M - 1, min(127, M - 1), min(128, M - 1)]])
            cols = np.concatenate([rng.integers(0, Nout, samples), [0, Nout - 1, 0, min(95, Nout - 1),
                                                                    min(192, Nout - 1)]])
            ref = self.y_ref_at(rows, cols)
            err = np.max(np.abs(y[rows, cols] - ref))
            # the bound is relative to max|y_ref| over all outputs; the max over the sampled outputs
            # is no larger, so using it is the stricter test
            scale = np.max(np.abs(ref))
        assert err <= REL_TOL * scale, f"max err {err:.3e} > {REL_TOL} * {scale:.3e}"
        return err / scale
