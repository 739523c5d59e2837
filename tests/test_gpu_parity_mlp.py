"""GPU checks of the MLP chain with the down layer's kernel 1 fused into the gate/up GEMM's SwiGLU
epilogue (svdq_gemm_swiglu_quant), against the oracle and against the unfused chain through the
same library (gemm with SwiGLU to a bf16 h, then svdq_quantize_act on h).

Against the oracle, on the h the GPU produced (the gate/up layer's own output is checked against
the oracle in test_gpu_parity.py): the down layer's activation scale, E2M1 codes, E4M3 scales and
alpha bit-exact against the oracle's calibration and quantization of h with the down layer's
smoothing; the down layer's fp32 output within 2e-3 of max|y_ref| of the oracle's layer forward on
h (every output, or a sample at full size).

Against the unfused chain: h bit-identical (when stored); codes, scales and alpha bit-identical
(the epilogue repeats kernel 1's arithmetic on the same bf16 h); U' within 1e-4 of max|U'| (fp32
sums over the 12288-wide K' in another order, then the same hi/lo split); the down layer's output
within 2e-4 of max|y|.
"""
import numpy as np
import pytest
import torch

import bit_diffusion_transformer_svdquant_b200 as svdq
from bit_diffusion_transformer_svdquant_b200 import synth
from oracle import svdquant

from _parity import REL_TOL, oracle_act_codes, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


def _rand(M, K, N, seed, bias, outlier=50.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, max(1, K // 100), replace=False)] *= outlier
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    b = svdquant.bf16_round(rng.standard_normal(N) * np.sqrt(0.02)) if bias else None
    return X, W, b


def _pack(X_cal, W, r, swiglu, dev):
    p = svdquant.prepare_layer(X_cal, W, r)
    w = svdq.PackedWeight(to_dev_f32(p["R"], dev), to_dev_bf16(p["L1s"], dev) if r else None,
                          to_dev_bf16(p["L2"], dev) if r else None, to_dev_f32(p["inv_lambda"], dev),
                          swiglu=swiglu)
    return w, p


def _check_against_oracle(h, prep_dn, b_dn, act_f, g_dn, y_f, samples):
    """The fused chain's down-layer quantization and output against the oracle on the GPU's h."""
    h_np = h.float().cpu().numpy().astype(np.float64)      # bf16 values, exact
    g_ref = svdquant.calibrate_activation_scale(h_np, prep_dn["inv_lambda"])
    assert float(g_dn.item()) == g_ref
    wq = svdquant.quantize_weight(prep_dn["R"])
    alpha_ref = float(np.float32(np.float32(g_ref) * np.float32(wq[0])))
    assert float(act_f.alpha().item()) == alpha_ref
    c_f, s_f = svdq.export_act(act_f)
    c_f, s_f = c_f.cpu().numpy(), s_f.cpu().numpy()
    c_ref, s_ref = oracle_act_codes(h_np, prep_dn["inv_lambda"], g_ref)
    assert np.array_equal(s_f, s_ref), np.argwhere(s_f != s_ref)[:10]
    assert np.array_equal(c_f, c_ref), np.argwhere(c_f != c_ref)[:10]
    y = y_f.cpu().numpy().astype(np.float64)
    assert np.isfinite(y).all()
    if samples is None:
        ref = svdquant.layer_forward(h_np, prep_dn, g_ref, wq, b_dn)
        err, scale = np.max(np.abs(y - ref)), np.max(np.abs(ref))
    else:
        M, N = y.shape
        rng = np.random.default_rng(7)
        rows = np.concatenate([rng.integers(0, M, samples), [0, M - 1, M - 1, min(128, M - 1)]])
        cols = np.concatenate([rng.integers(0, N, samples), [0, N - 1, 0, min(255, N - 1)]])
        ref = svdquant.layer_outputs_at(h_np, prep_dn, g_ref, wq, rows, cols, b_dn)
        err, scale = np.max(np.abs(y[rows, cols] - ref)), np.max(np.abs(ref))
    assert err <= REL_TOL * scale, f"max err {err:.3e} > {REL_TOL} * {scale:.3e}"


def _check_chain(X, W_up, b_up, r_up, X2_cal, W_dn, b_dn, r_dn, dev, samples=None):
    M = X.shape[0]
    w_up, _ = _pack(X, W_up, r_up, True, dev)
    w_dn, prep_dn = _pack(X2_cal, W_dn, r_dn, False, dev)
    Xd = to_dev_bf16(X, dev)
    bu = None if b_up is None else to_dev_bf16(b_up, dev)
    bd = None if b_dn is None else to_dev_bf16(b_dn, dev)
    g_up = svdq.calibrate_act(Xd, w_up)
    act_up = svdq.QuantizedAct(M, w_up.K, r_up, dev)
    svdq.quantize_act(Xd, w_up, g_up, act_up)
    # unfused: h to HBM, then kernel 1 of the down layer
    h = svdq.gemm(act_up, w_up, bu)
    g_dn = svdq.calibrate_act(h, w_dn)
    act_ref = svdq.QuantizedAct(M, w_dn.K, r_dn, dev)
    svdq.quantize_act(h, w_dn, g_dn, act_ref)
    # fused
    act_f = svdq.QuantizedAct(M, w_dn.K, r_dn, dev)
    h2 = torch.full_like(h, -7680.0)
    svdq.gemm_swiglu_quant(act_up, w_up, bu, w_dn, g_dn, act_f, h_out=h2)
    torch.cuda.synchronize(dev)
    assert svdq.device_status() == 0
    assert torch.equal(h2, h)
    c_ref, s_ref = svdq.export_act(act_ref)
    c_f, s_f = svdq.export_act(act_f)
    assert torch.equal(s_f, s_ref), torch.nonzero(s_f != s_ref)[:10]
    assert torch.equal(c_f, c_ref), torch.nonzero(c_f != c_ref)[:10]
    assert float(act_f.alpha().item()) == float(act_ref.alpha().item())
    u_ref = act_ref.U()[:, :M].float().sum(0)
    u_f = act_f.U()[:, :M].float().sum(0)
    assert float((u_f - u_ref).abs().max()) <= 1e-4 * float(u_ref.abs().max())
    y_ref = svdq.gemm(act_ref, w_dn, bd, out_dtype=torch.float32)
    y_f = svdq.gemm(act_f, w_dn, bd, out_dtype=torch.float32)
    torch.cuda.synchronize(dev)
    assert float((y_f - y_ref).abs().max()) <= 2e-4 * float(y_ref.abs().max())
    _check_against_oracle(h, prep_dn, b_dn, act_f, g_dn, y_f, samples)
    # the one-call chain (h never stored) gives the fused result
    y_mlp = svdq.mlp(Xd, w_up, g_up, w_dn, g_dn, bu, bd, out_dtype=torch.float32)
    torch.cuda.synchronize(dev)
    assert svdq.device_status() == 0
    assert torch.equal(y_mlp, y_f)


CASES = [
    # M, K, N_up (SwiGLU -> N_up / 2 = K of the down layer), N_down, r_up, r_down, bias
    (300, 512, 1024, 384, 16, 32, True),     # 4 column tiles, one per unit
    (1024, 256, 6144, 512, 32, 32, False),   # 24 column tiles in units of 3: U' accumulated across tiles
    (520, 512, 2560, 384, 32, 16, True),     # uneven units (1 or 2 tiles); an odd CTA past the last block
    (384, 256, 2048, 256, 0, 64, True),      # no branch in the gate/up layer; next rank 64
]


@pytest.mark.parametrize("M,K,N_up,N_dn,r_up,r_dn,bias", CASES)
def test_fused_chain_equals_unfused(cuda_device, M, K, N_up, N_dn, r_up, r_dn, bias):
    X, W_up, b_up = _rand(M, K, N_up, seed=M + N_up, bias=bias)
    X2, W_dn, b_dn = _rand(M, N_up // 2, N_dn, seed=M + N_dn + 1, bias=bias)
    _check_chain(X, W_up, b_up, r_up, X2, W_dn, b_dn, r_dn, cuda_device)


@pytest.mark.slow
def test_fused_chain_full_size_mlp_1024(cuda_device):
    """The 1024² MLP at full size (4608 tokens, 3072 -> 24576 SwiGLU -> 12288 -> 3072, r = 32)."""
    up, dn = synth.WORKLOADS["mlp_1024"].layers
    d_up, d_dn = synth.make_linear_inputs(up), synth.make_linear_inputs(dn)
    X, W_up = synth.bf16_values(d_up["X"]), synth.bf16_values(d_up["W"])
    X2, W_dn = synth.bf16_values(d_dn["X"]), synth.bf16_values(d_dn["W"])
    b_up = synth.bf16_values(d_up["bias"]) if up.bias else None
    b_dn = synth.bf16_values(d_dn["bias"]) if dn.bias else None
    _check_chain(X, W_up, b_up, up.r, X2, W_dn, b_dn, dn.r, cuda_device, samples=3000)
