"""OCP 8-bit floating point, E4M3 variant -- written from the OCP FP8 format
definition (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
infinities; the single NaN pattern per sign is S.1111.111; the largest finite
magnitude is 1.75 * 2^8 = 448; subnormals have exponent field 0 and value
m/8 * 2^-6).

The FP8 latent cache of the hotdry.top DeepSeek-V3 page ("支持 FP8 KV 缓存")
stores e4m3 codes with one fp32 scale per token.  Encoding rounds to the
nearest representable value, ties to even, and saturates finite values above
448 to +-448 (the "satfinite" convention: a cache entry must never become NaN
because of rounding).

Pinned by ``tests/test_oracle_e4m3.py``: all 256 codes decode to the values of
the format definition; every finite code round-trips; midpoints round to the
even neighbour; a large sweep agrees with ``torch``'s CPU float8_e4m3fn
conversion wherever that routine does not overflow; saturation and NaN.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6          # 2^-6 is the smallest normal magnitude
_MANT_BITS = 3


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 codes -> float64 values (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, _MIN_NORMAL_EXP)
    v = np.where(e == 0, sub, normal)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return v


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """float32 values -> uint8 e4m3 codes (round to nearest even, saturate to +-448).

    The input is taken as float32 (the precision in which the cache encoder
    makes its rounding decision); the rounding itself is done exactly in
    float64, where every float32 value and every e4m3 grid point is exact.
    """
    xf = np.asarray(x, dtype=np.float32)
    neg = np.signbit(xf)
    nan = np.isnan(xf)
    a = np.where(nan, 0.0, np.abs(xf).astype(np.float64))
    out = np.zeros(xf.shape, dtype=np.uint8)

    # exponent of the binade holding a (a = f * 2^k with f in [0.5, 1)), clamped
    # to the subnormal binade
    _, k = np.frexp(np.where(a > 0, a, 1.0))
    e = np.maximum(k - 1, _MIN_NORMAL_EXP)
    quantum = np.ldexp(1.0, (e - _MANT_BITS).astype(np.int64))
    n = np.rint(a / quantum)            # numpy rint: round half to even
    v = n * quantum                     # rounded magnitude, exact
    v = np.minimum(v, E4M3_MAX)         # satfinite

    # encode the rounded magnitude
    _, k2 = np.frexp(np.where(v > 0, v, 1.0))
    e2 = k2 - 1
    is_normal = v >= np.ldexp(1.0, _MIN_NORMAL_EXP)
    mant_n = np.rint((v / np.ldexp(1.0, e2.astype(np.int64)) - 1.0) * 8.0).astype(np.int64)
    code_n = ((e2 + 7) << 3) | mant_n
    code_s = np.rint(v / np.ldexp(1.0, _MIN_NORMAL_EXP - _MANT_BITS)).astype(np.int64)
    code = np.where(is_normal, code_n, code_s)
    code = np.where(v == 0, 0, code)
    out[...] = code.astype(np.uint8)
    out |= np.where(neg, 0x80, 0).astype(np.uint8)
    out[nan] = np.where(neg[nan], 0xFF, 0x7F).astype(np.uint8)
    return out
