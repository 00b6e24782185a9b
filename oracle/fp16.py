"""IEEE 754 binary16 from its definition (float64 in, float64 / uint16 out).

binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
  e == 0:        (-1)^s * f * 2^-24               (zero and subnormals)
  1 <= e <= 30:  (-1)^s * (1024 + f) * 2^(e - 25)
  e == 31:       infinity (f == 0) or NaN
Rounding is round-to-nearest, ties-to-even, applied once to the exact value.

The QTIP discussion fixes fp16 as the value type of its codebooks ("Bit
Accounting (Q2)": the HYB codebook takes 2^Q x V x 16 bits); the layer's
decoded weights are the fp16 rounding of each code value.
"""
from __future__ import annotations

import numpy as np

MAX_FINITE = 65504.0
_OVERFLOW = 65520.0  # halfway between 65504 and 2^16; ties go to the even 2^16 = inf


def decode_bits(bits) -> np.ndarray:
    """uint16 bit patterns -> exact float64 values."""
    b = np.asarray(bits).astype(np.int64) & 0xFFFF
    s = np.where(b >> 15, -1.0, 1.0)
    e = (b >> 10) & 31
    f = (b & 1023).astype(np.float64)
    out = np.where(e == 0, f * 2.0 ** -24, (1024.0 + f) * np.exp2((e - 25).astype(np.float64)))
    out = np.where(e == 31, np.where(f == 0, np.inf, np.nan), out)
    return s * out


def round_rne(v) -> np.ndarray:
    """Round float64 values to the nearest binary16 value, ties to even.

    Returns float64 values that are exactly representable in binary16
    (or +-inf on overflow). The sign of zero is preserved.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    mant, ex = np.frexp(np.where(a > 0, a, 1.0))  # a = mant * 2^ex, mant in [0.5, 1)
    e = np.maximum(ex - 1, -14)                    # exponent of the binade, clamped to the subnormal one
    quantum = np.exp2((e - 10).astype(np.float64))
    r = np.rint(a / quantum) * quantum              # np.rint: half to even; a/quantum is exact
    r = np.where(a == 0, 0.0, r)
    r = np.where(a >= _OVERFLOW, np.inf, r)
    r = np.where(np.isnan(v), np.nan, r)
    return np.copysign(r, v)


def encode(v) -> np.ndarray:
    """binary16-representable float64 values -> uint16 bit patterns."""
    v = np.asarray(v, dtype=np.float64)
    sign = np.signbit(v).astype(np.int64) << 15
    a = np.abs(v)
    mant, ex = np.frexp(np.where(a > 0, a, 1.0))
    e = ex - 1
    normal = e >= -14
    ef = np.where(normal, e + 15, 0)
    frac = np.where(normal, a / np.exp2(e.astype(np.float64)) * 1024.0 - 1024.0, a / 2.0 ** -24)
    bits = (ef << 10) | frac.astype(np.int64)
    bits = np.where(a == 0, 0, bits)
    bits = np.where(np.isinf(a), 31 << 10, bits)
    bits = np.where(np.isnan(v), 0x7E00, bits)
    if np.any(np.isfinite(a) & (frac != np.floor(frac))):
        raise ValueError("value not representable in binary16")
    return (bits | sign).astype(np.uint16)
