"""Pins of the oracle's NVFP4 block quantizer: invariants that the format and the rounding rules
fix, independent of how the oracle computes them."""
import numpy as np
import pytest

from oracle import nvfp4
from oracle.nvfp4 import f32


def _rand(rows, K, seed, outliers=True):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((rows, K))
    if outliers:
        v[:, rng.choice(K, max(1, K // 50), replace=False)] *= 50
    return f32(v)


def test_tensor_scale_definition():
    assert nvfp4.tensor_scale(2688.0) == 1.0
    assert nvfp4.tensor_scale(0.0) == 1.0
    assert nvfp4.tensor_scale(2.0 ** -101) == 1.0
    g = nvfp4.tensor_scale(10.0)
    assert g == float(np.float32(10.0 / 2688.0))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_amax_block_gets_largest_scale(seed):
    v = _rand(8, 256, seed)
    g = nvfp4.tensor_scale(np.abs(v).max())
    q, s = nvfp4.quantize(v, g)
    r, b = np.unravel_index(np.argmax(np.abs(v)), v.shape)
    assert s[r, b // 16] == 0x7E


@pytest.mark.parametrize("seed", [0, 1])
def test_block_max_encodes_to_six(seed):
    """For a normal, unsaturated scale, amax_b / (dec(s) g) lies within 6 * (1 +- 2^-4) (half an E4M3
    ulp), so the block's largest element always takes code +-6."""
    v = _rand(16, 512, seed)
    g = nvfp4.tensor_scale(np.abs(v).max())
    q, s = nvfp4.quantize(v, g)
    vb = v.reshape(16, 32, 16)
    normal = (s >= 0x08) & (s < 0x7E)
    ratio = np.abs(vb).max(axis=2) / (nvfp4.e4m3_decode(s) * g)
    assert np.all(ratio[normal] <= 6 * (1 + 2 ** -4) * (1 + 1e-6))
    assert np.all(ratio[normal] >= 6 / (1 + 2 ** -4) * (1 - 1e-6))
    imax = np.abs(vb).argmax(axis=2)
    qb = q.reshape(16, 32, 16)
    top = np.take_along_axis(qb, imax[:, :, None], axis=2)[:, :, 0]
    assert np.all((top[normal] & 7) == 7)


def test_idempotent_with_fixed_scales():
    v = _rand(16, 256, 4)
    g = nvfp4.tensor_scale(np.abs(v).max())
    q, s = nvfp4.quantize(v, g)
    d = nvfp4.dequantize(q, s, g)
    S = f32(nvfp4.e4m3_decode(s) * g)
    rS = f32(1.0 / np.where(s == 0, 1.0, S))
    q2 = nvfp4.e2m1_encode(f32(d.reshape(16, 16, 16) * rS[:, :, None])).reshape(16, 256)
    q2[np.repeat(s == 0, 16, axis=1)] = 0
    # +-0 both decode to 0; compare decoded codes and signs of nonzero ones
    assert np.array_equal(nvfp4.e2m1_decode(q2), nvfp4.e2m1_decode(q))
    nz = (q & 7) != 0
    assert np.array_equal(q2[nz], q[nz])


def test_zero_and_tiny_blocks():
    v = _rand(2, 64, 5)
    v[0, 16:32] = 0.0
    v[1, 0:16] = float(np.float32(1e-12))
    g = nvfp4.tensor_scale(np.abs(v).max())
    q, s = nvfp4.quantize(v, g)
    assert s[0, 1] == 0 and np.all(q[0, 16:32] == 0)
    assert s[1, 0] == 0 and np.all(q[1, 0:16] == 0)


def test_error_bound():
    """|v - dequant(v)| is at most half the local E2M1 spacing (<= 1 * dec(s) * g) plus the scale's
    own rounding; for normal scales the relative-to-block-amax error stays below 1/6 * 1.07."""
    v = _rand(32, 512, 6, outliers=False)
    g = nvfp4.tensor_scale(np.abs(v).max())
    q, s = nvfp4.quantize(v, g)
    d = nvfp4.dequantize(q, s, g)
    err = np.abs(d - v).reshape(32, 32, 16).max(axis=2)
    amax_b = np.abs(v).reshape(32, 32, 16).max(axis=2)
    assert np.all(err <= amax_b / 6 * 1.07 + 1e-30)


def test_static_scale_saturates():
    """A static scale calibrated on smaller data saturates scales at 448 and codes at 6."""
    v = _rand(1, 64, 8, outliers=False)
    g = nvfp4.tensor_scale(np.abs(v).max() / 100.0)
    q, s = nvfp4.quantize(v, g)
    assert np.all(s == 0x7E)
    assert np.all((q.reshape(4, 16) & 7).max(axis=1) == 7)
