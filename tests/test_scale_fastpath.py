"""Host check of the rule kernel 1 uses to get a block's E4M3 scale without a division on most
blocks: the quotient amax / d6 is taken as fp32(amax * fp32(1 / d6)) and the exact IEEE division is
used only when that product lies within 4 ulps of an E4M3 rounding boundary (fp32 mantissa bits
19..0 equal to 0x80000) or below 2^-6. The rule must give exactly E4M3(fp32(amax / d6)), the
oracle's scale, for every amax; checked here with fp32 arithmetic emulated in numpy on random
tensor scales and on amax values placed on and around every E4M3 rounding boundary."""
import numpy as np

from oracle import nvfp4
from oracle.nvfp4 import f32


def _fast_rule(amax, d6, rd6):
    q = f32(amax * rd6)
    bits = q.astype(np.float32).view(np.uint32).astype(np.int64)
    near = ((bits & 0xFFFFF) - 0x7FFFC) & 0xFFFFFFFF <= 8
    exact = f32(amax / d6)
    return np.where((q < 2.0 ** -6) | near, exact, q)


def _check(amax, g):
    d6 = float(f32(6.0 * g))
    rd6 = float(f32(1.0 / d6))
    want = nvfp4.e4m3_encode(f32(amax / d6))
    got = nvfp4.e4m3_encode(_fast_rule(amax, d6, rd6))
    bad = np.nonzero(want != got)[0]
    assert bad.size == 0, f"g={g}: amax {amax[bad[:5]]} -> {got[bad[:5]]}, want {want[bad[:5]]}"


def test_random_blocks():
    rng = np.random.default_rng(3)
    for _ in range(40):
        g = float(f32(rng.uniform(1e-4, 1.0) * 10.0 ** rng.integers(-6, 3)))
        amax = f32(np.abs(rng.standard_normal(200_000)) * g * 6 * 448 / 4)
        _check(amax, g)


def test_amax_on_and_around_every_rounding_boundary():
    rng = np.random.default_rng(4)
    mags = nvfp4._e4m3_magnitudes()
    mids = (mags[1:] + mags[:-1]) / 2
    for _ in range(20):
        g = float(f32(rng.uniform(1e-3, 1.0) * 10.0 ** rng.integers(-4, 2)))
        d6 = float(f32(6.0 * g))
        centre = f32(mids * d6)
        steps = np.arange(-12, 13)
        # amax values a few fp32 ulps around amax = midpoint * d6
        cand = []
        for k in steps:
            v = centre.astype(np.float32)
            for _ in range(abs(int(k))):
                v = np.nextafter(v, np.float32(np.inf if k > 0 else -np.inf))
            cand.append(v)
        amax = np.concatenate(cand).astype(np.float64)
        _check(amax[amax > 0], g)
