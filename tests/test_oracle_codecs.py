"""Pins of the oracle's E2M1 / E4M3 codecs against things other than the oracle itself.

1. Hand-derived fixed points of the formats (tests/golden/nvfp4_codes.txt).
2. A closed-form round-half-even formulation (scale to the binade's quantum, np.rint, saturate),
   which shares nothing with the oracle's table search, checked on every rounding boundary and its
   fp32 neighbours and on a dense sweep of fp32 bit patterns.
3. torch's float8_e4m3fn conversion (a library routine) for E4M3 below the saturation region.
4. Grid enumeration and monotonicity.
"""
import os

import numpy as np
import pytest
import torch

from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_codes.txt")


def _closed_form(a, min_exp, mant_bits, max_val):
    """|value| rounded half-even to the format's grid by scaling with the binade's quantum."""
    a = np.abs(np.asarray(a, dtype=np.float64))
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, min_exp)
    q = np.exp2(e - mant_bits)
    v = np.rint(a / q) * q
    return np.minimum(v, max_val)


def e2m1_closed(a):
    return _closed_form(a, 0, 1, 6.0)


def e4m3_closed(a):
    return _closed_form(a, -6, 3, 448.0)


def fp32_neighbours(points, k=3):
    pts = np.asarray(points, dtype=np.float32)
    out = [pts]
    up, dn = pts.copy(), pts.copy()
    for _ in range(k):
        up = np.nextafter(up, np.float32(np.inf))
        dn = np.nextafter(dn, np.float32(0))
        out += [up, dn]
    return np.concatenate(out).astype(np.float64)


def test_golden_fixed_points():
    n = 0
    with open(GOLDEN) as f:
        for line in f:
            if not line.strip() or line.startswith("#"):
                continue
            fmt, val, code = line.split()
            v = float(val)
            enc = nvfp4.e2m1_encode if fmt == "e2m1" else nvfp4.e4m3_encode
            got = int(enc(np.array([v]))[0])
            assert got == int(code, 16), (fmt, val, hex(got), code)
            n += 1
    assert n > 40


def test_e2m1_grid_enumeration():
    assert list(nvfp4.e2m1_decode(np.arange(8))) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(nvfp4.e2m1_decode(np.arange(8, 16))) == [-0.0, -0.5, -1, -1.5, -2, -3, -4, -6]
    # every code round-trips
    for c in range(16):
        assert int(nvfp4.e2m1_encode(nvfp4.e2m1_decode(np.array([c])))[0]) == c


def test_e4m3_grid_enumeration():
    mags = nvfp4.E4M3_MAGNITUDES
    assert mags.size == 127 and np.all(np.diff(mags) > 0)
    assert mags[0x7E] == 448.0 and mags[0x38] == 1.0 and mags[0x01] == 2.0 ** -9 and mags[0x08] == 2.0 ** -6
    codes = np.arange(0x7F, dtype=np.uint8)
    assert np.array_equal(nvfp4.e4m3_encode(nvfp4.e4m3_decode(codes)), codes)
    assert np.array_equal(nvfp4.e4m3_encode(-nvfp4.e4m3_decode(codes[1:])), codes[1:] | 0x80)


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_boundaries_against_closed_form(fmt):
    mags = nvfp4.E2M1_MAGNITUDES if fmt == "e2m1" else nvfp4.E4M3_MAGNITUDES
    enc = nvfp4.e2m1_encode if fmt == "e2m1" else nvfp4.e4m3_encode
    dec = nvfp4.e2m1_decode if fmt == "e2m1" else nvfp4.e4m3_decode
    closed = e2m1_closed if fmt == "e2m1" else e4m3_closed
    mids = (mags[:-1] + mags[1:]) / 2
    pts = fp32_neighbours(np.concatenate([mids, mags, [mags[-1] * 1.04, mags[-1] * 1.1, 1e30]]))
    pts = np.concatenate([pts, -pts])
    got = dec(enc(pts))
    want = np.copysign(closed(pts), pts)
    assert np.array_equal(got, want)
    assert np.array_equal(np.signbit(got), np.signbit(pts))


@pytest.mark.parametrize("fmt,hi_bits,stride", [("e2m1", 0x41000000, 37), ("e4m3", 0x43F00000, 61)])
def test_dense_fp32_sweep_against_closed_form(fmt, hi_bits, stride):
    """Every `stride`-th fp32 bit pattern from +0 up to 8.0 (E2M1) or 480.0 (E4M3)."""
    enc = nvfp4.e2m1_encode if fmt == "e2m1" else nvfp4.e4m3_encode
    dec = nvfp4.e2m1_decode if fmt == "e2m1" else nvfp4.e4m3_decode
    closed = e2m1_closed if fmt == "e2m1" else e4m3_closed
    for lo in range(0, hi_bits, 1 << 26):
        bits = np.arange(lo, min(lo + (1 << 26), hi_bits), stride, dtype=np.uint32)
        v = bits.view(np.float32).astype(np.float64)
        assert np.array_equal(dec(enc(v)), closed(v)), (fmt, hex(lo))


# Every rounding decision of E2M1 lies in [2^-3, 2^3) (below 0.25 all round to zero, above 6 all
# saturate) and every decision of E4M3 in [2^-11, 2^9) (below 2^-10 zero, above 464 saturation).
# These windows are checked for every fp32 bit pattern, one binade at a time; the tails are sampled.
DECISION_WINDOWS = {"e2m1": (-3, 3), "e4m3": (-11, 9)}


@pytest.mark.parametrize("fmt", ["e2m1", "e4m3"])
def test_every_fp32_in_decision_window(fmt):
    enc = nvfp4.e2m1_encode if fmt == "e2m1" else nvfp4.e4m3_encode
    dec = nvfp4.e2m1_decode if fmt == "e2m1" else nvfp4.e4m3_decode
    closed = e2m1_closed if fmt == "e2m1" else e4m3_closed
    top = 6.0 if fmt == "e2m1" else 448.0
    lo_e, hi_e = DECISION_WINDOWS[fmt]
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in range(lo_e, hi_e):
        bits = mant | np.uint32((e + 127) << 23)
        v32 = bits.view(np.float32)
        v = v32.astype(np.float64)
        codes = enc(v)
        assert np.array_equal(dec(codes), closed(v)), (fmt, e)
        if fmt == "e4m3":
            # torch's cast is not saturating (464 and above become NaN), so it is a second
            # formulation only below the saturation boundary.
            fin = v < 464.0
            ref = torch.from_numpy(v32[fin]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(codes[fin], ref), e
        neg = enc(-v[::7])
        sign = np.uint8(0x08 if fmt == "e2m1" else 0x80)
        assert np.array_equal(neg, codes[::7] | sign), (fmt, e)
    rng = np.random.default_rng(11)
    below = rng.integers(0, (lo_e + 127) << 23, 1 << 20, dtype=np.uint32).view(np.float32)
    above = rng.integers((hi_e + 127) << 23, 0x7F800000, 1 << 20, dtype=np.uint32).view(np.float32)
    assert np.all(dec(enc(below.astype(np.float64))) == 0.0)
    assert np.all(dec(enc(above.astype(np.float64))) == top)


def test_e4m3_against_torch_float8():
    rng = np.random.default_rng(7)
    v = np.concatenate([
        rng.uniform(0, 463.9, 2_000_000),
        np.exp2(rng.uniform(-14, 8.85, 2_000_000)),
        fp32_neighbours((nvfp4.E4M3_MAGNITUDES[:-1] + nvfp4.E4M3_MAGNITUDES[1:]) / 2)])
    v = v.astype(np.float32)
    v = np.concatenate([v, -v])
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = nvfp4.e4m3_encode(v.astype(np.float64))
    assert np.array_equal(got, ref)


def test_monotone():
    rng = np.random.default_rng(3)
    v = np.sort(rng.uniform(-500, 500, 1_000_000).astype(np.float32).astype(np.float64))
    for enc, dec in ((nvfp4.e2m1_encode, nvfp4.e2m1_decode), (nvfp4.e4m3_encode, nvfp4.e4m3_decode)):
        d = dec(enc(v))
        assert np.all(np.diff(d) >= 0)


def test_nibble_packing():
    c = np.arange(16, dtype=np.uint8).reshape(2, 8)
    p = nvfp4.pack_nibbles(c)
    assert p[0, 0] == 0x10 and p[0, 1] == 0x32 and p.shape == (2, 4)
    assert np.array_equal(nvfp4.unpack_nibbles(p), c)
