"""Pins of the oracle's smoothing, low-rank split and layer forward."""
from fractions import Fraction

import numpy as np
import pytest

from bit_diffusion_transformer_svdquant_b200 import synth
from oracle import nvfp4, svdquant


def _small(M=48, K=64, N=40, seed=0):
    rng = np.random.default_rng(seed)
    X = svdquant.bf16_round(rng.standard_normal((M, K)) * np.where(rng.random(K) < 0.05, 40, 1))
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    b = svdquant.bf16_round(rng.standard_normal(N) * 0.14)
    return X, W, b


def test_bf16_round():
    assert svdquant.bf16_round(1.0 + 2 ** -8) == 1.0              # tie -> even
    assert svdquant.bf16_round(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6
    assert svdquant.bf16_round(1.0 + 2 ** -8 + 2 ** -30) == 1.0 + 2 ** -7
    assert svdquant.bf16_round(-3.0) == -3.0


def test_bf16_round_against_torch():
    """torch's fp32 -> bf16 cast (a library routine, round-half-even) on random fp32 values over the
    normal range and on exact ties (low 16 bits 0x8000, both mantissa parities)."""
    import torch
    rng = np.random.default_rng(2)
    bits = rng.integers(0x00800000, 0x7F000000, 1_000_000, dtype=np.uint32)
    ties = (bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    sign = np.where(rng.random(bits.size) < 0.5, np.uint32(0x80000000), np.uint32(0))
    v32 = np.concatenate([bits | sign, ties | sign]).view(np.float32)
    ref = torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(svdquant.bf16_round(v32.astype(np.float64)), ref)


def test_smoothing_identity():
    X, W, _ = _small()
    inv, lam = svdquant.smoothing(X, W)
    lhs = X @ W.T
    rhs = (X * inv[None, :]) @ (lam[:, None] * W.T)
    assert np.max(np.abs(lhs - rhs)) <= 1e-12 * np.max(np.abs(lhs))
    # migration strength 1/2: smoothed column maxima of X and rows of W_hat coincide (up to inv's fp32 rounding)
    a = np.abs(X * inv).max(axis=0)
    b = np.abs(lam[:, None] * W.T).max(axis=1)
    assert np.allclose(a, b, rtol=2e-7)


def test_smoothing_zero_channel():
    X, W, _ = _small()
    X[:, 3] = 0.0
    W[:, 5] = 0.0
    inv, lam = svdquant.smoothing(X, W)
    assert inv[3] == 1.0 and inv[5] == 1.0


@pytest.mark.parametrize("r", [0, 4, 16])
def test_split_identity_and_eckart_young(r):
    X, W, _ = _small()
    p = svdquant.prepare_layer(X, W, r)
    W_hat = p["lam_prime"][:, None] * W.T
    recon = (p["lam_prime"][:, None] * p["L1s"]) @ p["L2"] + p["R"].T
    # only R's fp32 rounding separates the two
    assert np.all(np.abs(recon - W_hat) <= np.abs(p["R"].T) * 2 ** -24 + 1e-300)
    U, S, Vt = np.linalg.svd(W_hat, full_matrices=False)
    trunc = W_hat - (U[:, :r] * S[:r]) @ Vt[:r] if r else W_hat
    sig = np.linalg.norm(trunc, 2)
    assert abs(sig - S[r]) <= 1e-10 * S[0]
    if r == 0:
        assert np.array_equal(p["R"].T, nvfp4.f32(W_hat))


def _exact_layer(X, p, g_x, wq, bias):
    """Exact rational triple loop over the decoded codes, scales and branch weights."""
    g_w, wc, ws = wq
    xc, xs = svdquant.quantize_activations(X, p["inv_lambda"], g_x)
    xv = nvfp4.block_values(xc, xs)
    wv = nvfp4.block_values(wc, ws)
    M, K = X.shape
    N = wc.shape[0]
    r = p["r"]
    y = np.empty((M, N))
    gg = Fraction(g_x) * Fraction(g_w)
    for m in range(M):
        u = [sum(Fraction(X[m, k]) * Fraction(p["L1s"][k, j]) for k in range(K)) for j in range(r)]
        for n in range(N):
            acc = sum(Fraction(xv[m, k]) * Fraction(wv[n, k]) for k in range(K))
            lr = sum(u[j] * Fraction(p["L2"][j, n]) for j in range(r))
            y[m, n] = float(gg * acc + lr + (Fraction(bias[n]) if bias is not None else 0))
    return y


def test_layer_against_exact_triple_loop():
    X, W, b = _small(M=5, K=32, N=6, seed=3)
    p = svdquant.prepare_layer(X, W, 2)
    g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
    wq = svdquant.quantize_weight(p["R"])
    y = svdquant.layer_forward(X, p, g_x, wq, b)
    ye = _exact_layer(X, p, g_x, wq, b)
    assert np.max(np.abs(y - ye)) <= 1e-12 * np.max(np.abs(ye))


def test_rank_zero_is_plain_w4a4():
    X, W, b = _small(seed=4)
    p = svdquant.prepare_layer(X, W, 0)
    g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
    wq = svdquant.quantize_weight(p["R"])
    y = svdquant.layer_forward(X, p, g_x, wq, b)
    xq = svdquant.quantize_activations(X, p["inv_lambda"], g_x)
    plain = g_x * wq[0] * (nvfp4.dequantize(*xq, 1.0) @ nvfp4.dequantize(wq[1], wq[2], 1.0).T) + b
    assert np.max(np.abs(y - plain)) <= 1e-12 * np.max(np.abs(plain))


def test_swiglu_closed_form():
    z = np.array([0.0, 1.0, 40.0, -40.0, -800.0])
    s = svdquant.silu(z)
    assert s[0] == 0.0 and abs(s[1] - 1 / (1 + np.exp(-1))) < 1e-15
    assert abs(s[2] - 40.0) < 1e-12 and abs(s[3]) < 1e-15 and s[4] == 0.0
    y = np.array([[1.0, -2.0, 3.0, 0.5]])
    assert np.allclose(svdquant.apply_swiglu(y), [[svdquant.silu(1.0) * 3.0, svdquant.silu(-2.0) * 0.5]])


def test_sampled_outputs_match_full():
    X, W, b = _small(M=20, K=64, N=16, seed=5)
    p = svdquant.prepare_layer(X, W, 4)
    g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
    wq = svdquant.quantize_weight(p["R"])
    for sw in (False, True):
        y = svdquant.layer_forward(X, p, g_x, wq, b, swiglu=sw)
        rows = np.array([0, 3, 19, 7])
        cols = np.array([0, 5, 7, 2])
        ys = svdquant.layer_outputs_at(X, p, g_x, wq, rows, cols, b, swiglu=sw)
        assert np.allclose(ys, y[rows, cols], rtol=1e-13, atol=1e-13)


def test_quantized_layer_tracks_unquantized_on_tiny_workload():
    """Informational-quality sanity (not a parity gate): the W4A4 + low-rank layer stays close
    to the unquantized product, and the low-rank branch helps on outlier-heavy inputs."""
    spec = synth.WORKLOADS["tiny"].layers[0]
    d = synth.make_linear_inputs(spec)
    X, W = synth.bf16_values(d["X"]), synth.bf16_values(d["W"])
    ref = X @ W.T
    errs = {}
    for r in (0, spec.r):
        p = svdquant.prepare_layer(X, W, r)
        g_x = svdquant.calibrate_activation_scale(X, p["inv_lambda"])
        y = svdquant.layer_forward(X, p, g_x, svdquant.quantize_weight(p["R"]))
        errs[r] = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert errs[spec.r] < 0.2 and errs[spec.r] <= errs[0] * 1.05


def test_lora_on_the_branch_is_additive():
    """Concatenating a LoRA adapter onto the branch adds exactly X A B to the layer output (the
    linearity the reading relies on), and r grows by the adapter rank."""
    rng = np.random.default_rng(7)
    M, K, N = 24, 64, 48
    X = svdquant.bf16_round(rng.standard_normal((M, K)))
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / 8)
    prep = svdquant.prepare_layer(X, W, 16)
    A = svdquant.bf16_round(rng.standard_normal((K, 16)) / 8)
    B = svdquant.bf16_round(rng.standard_normal((16, N)) / 8)
    lp = svdquant.add_lora(prep, A, B)
    assert lp["r"] == 32 and lp["L1s"].shape == (K, 32) and lp["L2"].shape == (32, N)
    g_x = svdquant.calibrate_activation_scale(X, prep["inv_lambda"])
    wq = svdquant.quantize_weight(prep["R"])
    base = svdquant.layer_forward(X, prep, g_x, wq)
    with_lora = svdquant.layer_forward(X, lp, g_x, wq)
    np.testing.assert_allclose(with_lora, base + (X @ A) @ B, rtol=1e-12, atol=1e-12)
    # a rank-0 layer plus an adapter is the adapter alone on top of plain W4A4
    p0 = svdquant.prepare_layer(X, W, 0)
    wq0 = svdquant.quantize_weight(p0["R"])
    l0 = svdquant.add_lora(p0, A, B)
    np.testing.assert_allclose(svdquant.layer_forward(X, l0, g_x, wq0),
                               svdquant.layer_forward(X, p0, g_x, wq0) + (X @ A) @ B, rtol=1e-12, atol=1e-12)


def test_activation_scale_on_a_hand_example():
    """The static activation scale is taken over the SMOOTHED activations: g_x = fp32(max|x *
    inv_lambda| / 2688). Hand example (4 tokens x 32 channels, bf16-exact values): channel 3 is an
    outlier channel (raw values up to 100) with inv_lambda = 1/4, so its smoothed values peak at 25;
    channel 21 holds the smoothed maximum, x = -40 with inv_lambda = 1. So the smoothed amax is 40,
    the raw amax 100, and the block of 16 channels holding (token 2, channel 21) is the one whose
    E4M3 scale is 448 (code 0x7E). A scale computed on the unsmoothed X (100 / 2688) or with lambda
    in place of 1 / lambda (100 * 4 / 2688) gives another value, so either mistake fails here."""
    X = np.zeros((4, 32))
    X[:, 0] = [1.5, -2.0, 0.5, 3.0]
    X[:, 3] = [100.0, -96.0, 64.0, 80.0]
    X[:, 21] = [12.0, 8.0, -40.0, 30.0]
    X[:, 30] = [-6.0, 7.0, 2.0, -3.5]
    inv_lambda = np.ones(32)
    inv_lambda[3] = 0.25
    inv_lambda[30] = 0.5
    g_expected = float(np.float32(40.0 / 2688.0))
    g = svdquant.calibrate_activation_scale(X, inv_lambda)
    assert g == g_expected
    assert g != float(np.float32(100.0 / 2688.0))        # raw amax
    assert g != float(np.float32(400.0 / 2688.0))        # lambda instead of 1 / lambda
    q, s = svdquant.quantize_activations(X, inv_lambda, g)
    assert s.shape == (4, 2)
    assert s[2, 1] == 0x7E                                # block (token 2, channels 16..31)
    assert (s[[0, 1, 3], 1] < 0x7E).all() and (s[:, 0] < 0x7E).all()
    # the amax element itself encodes to -6 (sign bit | code 7)
    assert q[2, 21] == 0x8 | 0x7
