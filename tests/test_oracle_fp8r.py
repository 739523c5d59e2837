"""Pins of the row-wise FP8 (W8A8) oracle: properties the format's definition fixes, checked
independently of the oracle's own arithmetic (fixed-scale idempotence, the amax element, zero rows,
the E4M3 spacing bound, power-of-two scale invariance, an exact-rational layer)."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import fp8r, nvfp4, svdquant


def _rows(seed, rows=64, K=96, outliers=True):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, K))
    if outliers:
        v[:, :3] *= 40.0
    v[rows // 2] *= 1e-3
    return nvfp4.f32(v)


def test_fixed_scale_idempotence():
    v = _rows(1)
    s, q = fp8r.quantize_rows(v)
    back = fp8r.dequantize_rows(s, q)
    # requantize the decoded values with the scales held fixed: the same codes
    q2 = nvfp4.e4m3_encode(nvfp4.f32(back * nvfp4.f32(1.0 / s)[:, None]))
    assert np.array_equal(q, q2)


def test_amax_element_lands_on_448():
    v = _rows(2)
    s, q = fp8r.quantize_rows(v)
    i = np.abs(v).argmax(axis=1)
    top = q[np.arange(v.shape[0]), i]
    assert np.all((top & 0x7F) == 0x7E)          # magnitude code of 448
    assert np.all((top >> 7) == (v[np.arange(v.shape[0]), i] < 0))
    assert np.all(np.abs(fp8r.dequantize_rows(s, q)).max(axis=1) == 448.0 * s)


def test_zero_and_tiny_rows():
    v = np.zeros((3, 32))
    v[1, 5] = 2.0 ** -120
    s, q = fp8r.quantize_rows(v)
    assert np.all(s == 1.0)
    assert np.all((q & 0x7F) == 0)


def test_e4m3_spacing_bound():
    """Every code is within half the E4M3 spacing of the scaled fp32 value it encodes."""
    v = _rows(3)
    s, q = fp8r.quantize_rows(v)
    t = np.abs(nvfp4.f32(v * nvfp4.f32(1.0 / s)[:, None]))
    e = np.floor(np.log2(np.maximum(t, 2.0 ** -30)))
    spacing = np.where(t >= 2.0 ** -6, 2.0 ** (e - 3), 2.0 ** -9)
    err = np.abs(np.abs(nvfp4.e4m3_decode(q)) - np.minimum(t, 448.0))
    assert np.all(err <= spacing / 2)


@pytest.mark.parametrize("k", [-7, -1, 3, 11])
def test_power_of_two_scale_invariance(k):
    v = _rows(4, outliers=False)
    s, q = fp8r.quantize_rows(v)
    s2, q2 = fp8r.quantize_rows(v * 2.0 ** k)
    assert np.array_equal(q, q2)
    np.testing.assert_array_equal(s2, s * 2.0 ** k)


def _small_layer(seed, r, bias):
    rng = np.random.default_rng(seed)
    M, K, N = 5, 32, 6
    X = svdquant.bf16_round(rng.standard_normal((M, K)) * np.where(np.arange(K) < 2, 30.0, 1.0))
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / 6)
    b = svdquant.bf16_round(rng.standard_normal(N) * 0.1) if bias else None
    return X, W, b, svdquant.prepare_layer(X, W, r)


@pytest.mark.parametrize("r,bias", [(0, False), (4, True)])
def test_layer_exact_rational(r, bias):
    X, W, b, prep = _small_layer(5, r, bias)
    wq = fp8r.quantize_weight(prep["R"])
    y = fp8r.layer_forward(X, prep, wq, b)
    sx, qx = fp8r.quantize_activations(X, prep["inv_lambda"])
    dx, dw = nvfp4.e4m3_decode(qx), nvfp4.e4m3_decode(wq[1])
    M, K = X.shape
    N = W.shape[0]
    for m in range(M):
        for n in range(N):
            acc = sum(Fraction(float(dx[m, k])) * Fraction(float(dw[n, k])) for k in range(K))
            ref = Fraction(float(sx[m])) * Fraction(float(wq[0][n])) * acc
            if r:
                u = [sum(Fraction(float(X[m, k])) * Fraction(float(prep["L1s"][k, j])) for k in range(K))
                     for j in range(r)]
                ref += sum(u[j] * Fraction(float(prep["L2"][j, n])) for j in range(r))
            if bias:
                ref += Fraction(float(b[n]))
            assert abs(float(ref) - y[m, n]) <= 1e-12 * max(1.0, abs(float(ref)))


def test_r0_is_plain_w8a8():
    X, W, _, prep = _small_layer(6, 0, False)
    wq = fp8r.quantize_weight(prep["R"])
    sx, qx = fp8r.quantize_activations(X, prep["inv_lambda"])
    plain = (sx[:, None] * nvfp4.e4m3_decode(qx)) @ (wq[0][:, None] * nvfp4.e4m3_decode(wq[1])).T
    np.testing.assert_allclose(fp8r.layer_forward(X, prep, wq), plain, rtol=1e-13, atol=1e-13)


def test_branch_hi_lo_scheme_precision():
    """Precision budget of how the row-wise FP8 kernels carry the branch (a design check, emulated in
    fp64 with the kernels' explicit roundings): U / s_x and L2^T / s_w as bf16 hi/lo pairs, three
    products (hi.hi, lo.hi, hi.lo) accumulated with the FP8 product, then times s_x s_w. Its error
    against the exact (X L1s) L2 stays below 1e-4 of max|y| on an outlier-heavy layer, far inside
    the 2e-3 bar."""
    f32 = nvfp4.f32
    rng = np.random.default_rng(9)
    M, K, N, r = 256, 1024, 512, 32
    X = rng.standard_normal((M, K))
    X[:, rng.choice(K, 10, replace=False)] *= 50
    X = svdquant.bf16_round(X)
    W = svdquant.bf16_round(rng.standard_normal((N, K)) / np.sqrt(K))
    prep = svdquant.prepare_layer(X, W, r)
    s_w, q_w = fp8r.quantize_weight(prep["R"])
    s_x, _ = fp8r.quantize_activations(X, prep["inv_lambda"])
    y = fp8r.layer_forward(X, prep, (s_w, q_w))
    U = f32(X @ prep["L1s"])                                    # fp32 accumulate on the tensor cores
    u = f32(U * f32(1.0 / s_x)[:, None])
    u_hi = svdquant.bf16_round(u)
    u_lo = svdquant.bf16_round(f32(u - u_hi))
    v = f32(prep["L2"].T * f32(1.0 / s_w)[:, None])             # [N, r]
    l_hi = svdquant.bf16_round(v)
    l_lo = svdquant.bf16_round(f32(v - l_hi))
    acc = u_hi @ l_hi.T + u_lo @ l_hi.T + u_hi @ l_lo.T
    branch = f32(s_x[:, None] * s_w[None, :]) * acc
    exact = (X @ prep["L1s"]) @ prep["L2"]
    err = np.max(np.abs(branch - exact))
    assert err <= 1e-4 * np.max(np.abs(y)), err / np.max(np.abs(y))
    # without L2's lo half (U still hi/lo) the error is ~2^-9 relative to the branch: more than a
    # hundred times larger, about the size of the whole bar on this layer
    two = f32(s_x[:, None] * s_w[None, :]) * (u_hi @ l_hi.T + u_lo @ l_hi.T)
    assert np.max(np.abs(two - exact)) > 100 * err
