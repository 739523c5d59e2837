"""GPU parity of the row-wise FP8 (W8A8) variant (through the C ABI) against ``oracle/fp8r.py``.

Bar, as for the NVFP4 path: row scales and E4M3 codes bit-exact; fp32 outputs within
max|y - y_ref| <= 2e-3 * max|y_ref|; bf16 outputs bitwise equal to the bf16 rounding of the fp32
outputs. The low-rank branch runs as bf16 hi/lo pairs of U / s_x and L2^T / s_w (about 16
significant bits each), well inside that bar.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_svdquant_b200 as svdq
from oracle import fp8r, nvfp4, svdquant

from _parity import REL_TOL, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def _rand_layer(M, K, N, r, seed, bias=True, outlier=50.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, max(1, K // 100), replace=False)] *= outlier
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    b = svdquant.bf16_round(rng.standard_normal(N) * np.sqrt(0.02)) if bias else None
    return X, W, b


def _run(X, W, b, r, swiglu, dev, prep=None):
    prep = svdquant.prepare_layer(X, W, r) if prep is None else prep
    w = svdq.Fp8rWeight(to_dev_f32(prep["R"], dev), to_dev_bf16(prep["L1s"], dev) if r else None,
                        to_dev_bf16(prep["L2"], dev) if r else None, to_dev_f32(prep["inv_lambda"], dev),
                        swiglu=swiglu)
    act = svdq.Fp8rAct(X.shape[0], X.shape[1], r, dev)
    svdq.quantize_act_fp8r(to_dev_bf16(X, dev), w, act)
    return prep, w, act


def _check_codes(X, prep, w, act):
    s_w, q_w = fp8r.quantize_weight(prep["R"])
    c, s = svdq.export_weight_fp8r(w)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), s_w), "weight row scales differ"
    c = c.cpu().numpy()
    bad = np.argwhere(c != q_w)[:10]
    assert bad.size == 0, f"weight codes differ at {bad}"
    s_x, q_x = fp8r.quantize_activations(X, prep["inv_lambda"])
    c, s = svdq.export_act_fp8r(act)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), s_x), "activation row scales differ"
    c = c.cpu().numpy()
    bad = np.argwhere(c != q_x)[:10]
    assert bad.size == 0, (f"activation codes differ at {bad}: got {[hex(c[tuple(i)]) for i in bad]} "
                           f"want {[hex(q_x[tuple(i)]) for i in bad]}")
    return (s_w, q_w)


def _check_outputs(X, prep, wq, b, swiglu, w, act, dev):
    bias_d = None if b is None else to_dev_bf16(b, dev)
    y32 = svdq.gemm_fp8r(act, w, bias_d, out_dtype=torch.float32)
    ybf = svdq.gemm_fp8r(act, w, bias_d, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert svdq.device_status() == 0
    assert torch.equal(ybf, y32.to(torch.bfloat16))
    y = y32.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    ref = fp8r.layer_forward(X, prep, wq, b, swiglu)
    err, scale = np.max(np.abs(y - ref)), np.max(np.abs(ref))
    assert err <= REL_TOL * scale, f"max err {err:.3e} > {REL_TOL} * {scale:.3e}"


CASES = [
    # M, K, N, r, bias, swiglu      (tile width: 256 where it divides N, else 192, else 128)
    (300, 768, 384, 32, True, False),   # ragged M (odd number of 128-row blocks), 192-wide tiles
    (1, 256, 128, 0, False, False),     # one row, no branch, 128-wide tile
    (200, 512, 768, 64, True, True),    # SwiGLU with bias, r = 64, 256-wide tiles
    (513, 256, 256, 16, False, False),  # a ragged fifth row block, one K step pair, r = 16
    (257, 512, 640, 32, True, True),    # SwiGLU on 128-wide tiles
]


@pytest.mark.parametrize("M,K,N,r,bias,swiglu", CASES)
def test_fp8r_small_shapes(cuda_device, M, K, N, r, bias, swiglu):
    X, W, b = _rand_layer(M, K, N, r, seed=M * 11 + N, bias=bias)
    prep, w, act = _run(X, W, b, r, swiglu, cuda_device)
    wq = _check_codes(X, prep, w, act)
    _check_outputs(X, prep, wq, b, swiglu, w, act, cuda_device)


def test_fp8r_codec_edges(cuda_device):
    """With lambda = 1 and a row whose amax is 448, s_x = 1 and the codes are the E4M3 rounding of the
    values themselves: ties between grid points, values that round to zero with either sign, a zero
    row (s_x = 1) and a row below the tiny-amax threshold."""
    K, M = 256, 8
    rng = np.random.default_rng(5)
    X = svdquant.bf16_round(rng.standard_normal((M, K)))
    ties = [1.0625, 1.1875, 3.0 * 2.0 ** -9 / 2, 2.0 ** -10, -2.0 ** -10, 2.0 ** -11, -2.0 ** -11, 240.0, 464.0 / 2]
    X[1, :] = 0.0
    X[1, 0] = 448.0
    X[1, 1:1 + len(ties)] = ties
    X[2, :] = 0.0
    X[3, :] = 2.0 ** -110
    X[3, ::2] *= -1
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((128, K)) / 16)
    prep = {"inv_lambda": np.ones(K), "lam_prime": np.ones(K), "L1s": np.zeros((K, 0)), "L2": np.zeros((0, 128)),
            "R": nvfp4.f32(W), "r": 0}
    prep_, w, act = _run(X, W, None, 0, False, cuda_device, prep=prep)
    wq = _check_codes(X, prep_, w, act)
    _check_outputs(X, prep_, wq, None, False, w, act, cuda_device)


MULTI_TILE = [
    # more tiles than resident CTA pairs: accumulator double-buffering and the ring / relay
    # barrier phases carried from one tile to the next
    (2048, 512, 9216, 32, True, False),   # 256-wide tiles, ~4 per pair
    (1024, 256, 6144, 16, False, True),   # SwiGLU on 256-wide tiles
    (1536, 256, 5760, 32, True, False),   # 192-wide tiles (30 column blocks)
    (1280, 256, 4736, 64, True, True),    # 128-wide tiles (37 column blocks), SwiGLU, r = 64
]


@pytest.mark.parametrize("M,K,N,r,bias,swiglu", MULTI_TILE)
def test_fp8r_multi_tile(cuda_device, M, K, N, r, bias, swiglu):
    X, W, b = _rand_layer(M, K, N, r, seed=M + 7 * N, bias=bias)
    prep, w, act = _run(X, W, b, r, swiglu, cuda_device)
    wq = _check_codes(X, prep, w, act)
    _check_outputs(X, prep, wq, b, swiglu, w, act, cuda_device)


def _full_layers():
    from bit_diffusion_transformer_svdquant_b200 import synth
    return [pytest.param(spec, id=spec.name) for name in ("qkv_2048", "mlp_1024")
            for spec in synth.WORKLOADS[name].layers]


@pytest.mark.slow
@pytest.mark.parametrize("spec", _full_layers())
def test_fp8r_full_size_sampled_rows(cuda_device, spec):
    """Full-size layers. Token rows are independent in this variant (each has its own scale), so
    the oracle's values on a row sample are exact: all weight codes and scales, the sampled rows'
    activation codes and scales, and their outputs within tolerance; bf16 = bf16(fp32) everywhere."""
    from bit_diffusion_transformer_svdquant_b200 import synth
    d = synth.make_linear_inputs(spec)
    X, W = synth.bf16_values(d["X"]), synth.bf16_values(d["W"])
    b = synth.bf16_values(d["bias"]) if spec.bias else None
    prep, w, act = _run(X, W, b, spec.r, spec.swiglu, cuda_device)
    s_w, q_w = fp8r.quantize_weight(prep["R"])
    c, s = svdq.export_weight_fp8r(w)
    assert np.array_equal(s.cpu().numpy().astype(np.float64), s_w)
    assert np.array_equal(c.cpu().numpy(), q_w)
    M = X.shape[0]
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([rng.choice(M, 200, replace=False), [0, 127, 128, 255, 256, M - 1]]))
    s_x, q_x = fp8r.quantize_activations(X[rows], prep["inv_lambda"])
    c, s = svdq.export_act_fp8r(act)
    assert np.array_equal(s.cpu().numpy()[rows].astype(np.float64), s_x)
    assert np.array_equal(c.cpu().numpy()[rows], q_x)
    bias_d = None if b is None else to_dev_bf16(b, cuda_device)
    y32 = svdq.gemm_fp8r(act, w, bias_d, out_dtype=torch.float32)
    ybf = svdq.gemm_fp8r(act, w, bias_d, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert svdq.device_status() == 0
    assert torch.equal(ybf, y32.to(torch.bfloat16))
    y = y32.cpu().numpy()[rows].astype(np.float64)
    ref = fp8r.layer_forward(X[rows], prep, (s_w, q_w), b, spec.swiglu)
    err, scale = np.max(np.abs(y - ref)), np.max(np.abs(ref))
    assert err <= REL_TOL * scale, f"max err {err:.3e} > {REL_TOL} * {scale:.3e}"
