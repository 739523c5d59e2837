"""NVFP4 codecs and block quantizer (oracle; test infrastructure only, see ``oracle/__init__``).

Format. NVFP4 stores a tensor as 4-bit E2M1 codes, one E4M3 scale per 16 consecutive elements
along the reduction dimension K, and one fp32 scale for the whole tensor. The pages name the format
(FLUX 3 Image Klein on NVIDIA Blackwell, "Method 1: quantization (NVFP4 / FP8)"); the layout above is
the format's definition as used by this layer. Which steps round where is not on the pages; the
readings taken here are:

  * every named rounding is IEEE fp32 round-to-nearest-even, written here as "fp64 operation, then
    cast to float32" (exact for a single +, -, *, / of fp32 operands, since 53 >= 2*24 + 2);
  * E2M1 and E4M3 encodings round to nearest with ties to the even code and saturate at the
    largest finite magnitude (6 and 448); the sign is kept even when the magnitude rounds to 0;
  * tensor scale g = fp32(amax / (6 * 448)); a tensor whose amax is below 2**-100 (zero included)
    gets g = 1, which keeps every later reciprocal finite;
  * per block: s = E4M3(fp32(amax_b / fp32(6 g))); if s encodes 0 the 16 codes are +0; otherwise
    S = fp32(dec(s) * g), rS = fp32(1 / S), q_k = E2M1(fp32(v_k * rS)).
  * decoded value of element k: dec(q_k) * dec(s) * g.
"""
from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0
G_DIVISOR = E2M1_MAX * E4M3_MAX        # 2688
TINY_AMAX = 2.0 ** -100
BLOCK = 16

# E2M1 magnitudes by 3-bit magnitude code (sign is bit 3): 1 sign, 2 exponent (bias 1), 1 mantissa.
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _e4m3_magnitudes() -> np.ndarray:
    """E4M3 ("fn" variant) magnitudes by 7-bit code 0x00..0x7E; 0x7F is NaN and never produced."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        out.append(m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(out)


E4M3_MAGNITUDES = _e4m3_magnitudes()


def f32(x) -> np.ndarray:
    """Round fp64 value(s) to fp32 (IEEE round-to-nearest-even) and return them as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def _encode(v, magnitudes: np.ndarray, sign_bit: int) -> np.ndarray:
    """Nearest magnitude in the sorted table, ties to the even code, saturating; sign kept."""
    v = np.asarray(v, dtype=np.float64)
    if np.isnan(v).any():
        raise ValueError("NaN has no encoding here")
    a = np.abs(v)
    mids = (magnitudes[:-1] + magnitudes[1:]) / 2.0          # exact in fp64
    idx = np.searchsorted(mids, a, side="left")             # number of midpoints strictly below a
    at_mid = np.zeros(a.shape, dtype=bool)
    inside = idx < mids.size
    at_mid[inside] = a[inside] == mids[idx[inside]]
    idx = np.where(at_mid & (idx % 2 == 1), idx + 1, idx)   # tie between codes i, i+1: take the even one
    sign = np.signbit(v).astype(np.uint8)
    return (sign << sign_bit) | idx.astype(np.uint8)


def e2m1_encode(v) -> np.ndarray:
    """4-bit E2M1 codes (uint8 0..15, bit 3 = sign) of fp64 value(s)."""
    return _encode(v, E2M1_MAGNITUDES, 3)


def e2m1_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_encode(v) -> np.ndarray:
    """8-bit E4M3 codes (bit 7 = sign) of fp64 value(s), saturating at 448."""
    return _encode(v, E4M3_MAGNITUDES, 7)


def e4m3_decode(codes) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.uint8)
    if ((codes & 0x7F) == 0x7F).any():
        raise ValueError("E4M3 NaN code")
    mag = E4M3_MAGNITUDES[codes & 0x7F]
    return np.where(codes & 0x80, -mag, mag)


def tensor_scale(amax: float) -> float:
    """fp32 tensor scale g of a tensor whose largest magnitude is ``amax``."""
    amax = float(amax)
    if amax < TINY_AMAX:
        return 1.0
    return float(f32(amax / G_DIVISOR))


def quantize(v32: np.ndarray, g: float):
    """NVFP4 block quantization of the rows of ``v32`` (fp32 values, shape [rows, K], K % 16 == 0).

    Returns (codes uint8 [rows, K] one code per element, scales uint8 [rows, K/16]).
    """
    v = np.asarray(v32, dtype=np.float64)
    if not np.array_equal(f32(v), v):
        raise ValueError("quantize expects fp32-representable values")
    rows, K = v.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    vb = v.reshape(rows, K // BLOCK, BLOCK)
    amax_b = np.abs(vb).max(axis=2)
    d6 = f32(6.0 * g)
    s = e4m3_encode(f32(amax_b / d6))
    S = f32(e4m3_decode(s) * g)
    zero = s == 0
    rS = f32(1.0 / np.where(zero, 1.0, S))
    q = e2m1_encode(f32(vb * rS[:, :, None]))
    q[zero] = 0
    return q.reshape(rows, K), s


def dequantize(codes: np.ndarray, scales: np.ndarray, g: float) -> np.ndarray:
    """dec(q) * dec(s) * g for every element, fp64 (exact: every factor is a short binary fraction)."""
    rows, K = codes.shape
    d = e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK) * e4m3_decode(scales)[:, :, None]
    return d.reshape(rows, K) * g


def block_values(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """dec(q) * dec(s) without the tensor scale (what the block-scaled MMA multiplies)."""
    rows, K = codes.shape
    d = e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK) * e4m3_decode(scales)[:, :, None]
    return d.reshape(rows, K)


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte along the last axis: element 2i in the low nibble, 2i+1 in the high one."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
