"""FP8 E4M3 rounding, fp64 (the storage format of an fp8 K/V history).

TEST INFRASTRUCTURE, NOT PRODUCT CODE (see oracle/__init__.py).

Forcing-KV's reading notes report the method combined with FP8 on LongLive
(results, "LongLive + FP8 + Forcing-KV").  The pages do not say which tensors are
held in FP8 or in which encoding; the reading here is the retained K/V history
stored in the E4M3 encoding of FP8: 1 sign bit, 4 exponent bits with bias 7, 3
mantissa bits, subnormals below 2^-6 in steps of 2^-9, no infinities, the
all-ones code (S.1111.111) a NaN, so the largest finite magnitude is
1.75 * 2^8 = 448.  A value is rounded to the nearest representable one, ties to
the even mantissa, and magnitudes beyond 448 saturate to 448.

Pins: ``tests/test_oracle_fp8.py`` (hand values from the format, and a brute-force
nearest-code search over every decoded code).
"""
from __future__ import annotations

import numpy as np

MAX_E4M3 = 448.0


def e4m3(x) -> np.ndarray:
    """Round every element of x to the nearest E4M3 value (ties to even,
    saturating at +-448); returns float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    # binade exponent e with 2^e <= a < 2^(e+1); subnormals share e = -6
    _, E = np.frexp(np.maximum(a, 2.0 ** -6))
    e = E.astype(np.float64) - 1.0
    step = 2.0 ** (e - 3.0)                 # 3 mantissa bits
    q = np.round(a / step) * step            # numpy rounds halves to even
    q = np.minimum(q, MAX_E4M3)
    return np.where(x < 0, -q, q)


def decode_e4m3(code: int) -> float:
    """The value of an 8-bit E4M3 code (NaN for S.1111.111), from the bit layout."""
    s = -1.0 if (code >> 7) & 1 else 1.0
    ef = (code >> 3) & 0xF
    mf = code & 0x7
    if ef == 0xF and mf == 0x7:
        return float("nan")
    if ef == 0:
        return s * (mf / 8.0) * 2.0 ** -6
    return s * (1.0 + mf / 8.0) * 2.0 ** (ef - 7)
