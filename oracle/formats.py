"""Number-format rounding for the oracle (test infrastructure only).

All arithmetic is float64 numpy.  A value of a narrow format is carried as the
float64 number it represents.

Why float64 suffices for fp32 results: for one IEEE operation (+, -, *, /) on
fp32 operands, rounding the exact result first to float64 and then to fp32
gives the correctly rounded fp32 result, because 53 >= 2*24 + 2.  Products of
two fp32 numbers are even exact in float64.  So "compute in float64, then fl32"
is the fp32 operation itself.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32
F64 = np.float64


def fl32(v) -> np.ndarray:
    """Round float64 to the nearest fp32 (ties to even), returned as float64."""
    return np.asarray(v, dtype=F64).astype(F32).astype(F64)


def round_to_precision(v, p: int, emin: int, max_finite: float, saturate: bool) -> np.ndarray:
    """Round float64 values to a binary format with p significand bits.

    p counts the implicit bit; emin is the exponent of the smallest normal
    number (subnormals share its quantum).  Ties go to even.  Values whose
    rounded magnitude exceeds max_finite saturate to +-max_finite when
    `saturate`, else become +-inf.  NaN stays NaN.
    """
    v = np.asarray(v, dtype=F64)
    out = np.empty_like(v)
    a = np.abs(v)
    nan = np.isnan(v)
    # exponent of each value: a = m * 2**e with m in [1, 2)
    with np.errstate(divide="ignore"):
        _, e2 = np.frexp(a)          # a = f * 2**e2, f in [0.5, 1)
    e = e2.astype(np.int64) - 1
    e = np.maximum(e, emin)
    quantum = np.ldexp(np.ones_like(a), (e - (p - 1)).astype(np.int64))
    r = np.rint(a / quantum) * quantum   # a/quantum is exact (power-of-two scale)
    over = r > max_finite
    if saturate:
        r = np.where(over, max_finite, r)
    else:
        r = np.where(over, np.inf, r)
    r = np.where(np.isinf(a), np.inf if not saturate else max_finite, r)
    out[...] = np.copysign(r, v)
    out[nan] = np.nan
    return out


BF16_MAX = float(np.ldexp(2.0 - 2.0 ** -7, 127))


def bf16(v) -> np.ndarray:
    """Round to bfloat16 (8 significand bits, fp32 exponent range), ties to even."""
    return round_to_precision(v, 8, -126, BF16_MAX, saturate=False)


def bf16_bits(v) -> np.ndarray:
    """uint16 encoding of values already representable in bf16."""
    f = np.asarray(v, dtype=F64).astype(F32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    u = np.asarray(b, dtype=np.uint32) << 16
    return u.astype(np.uint32).view(F32).astype(F64)


def f32_bits(v) -> np.ndarray:
    return np.asarray(v, dtype=F64).astype(F32).view(np.uint32)


# ---------------------------------------------------------------- E4M3 (OCP FP8)
# QLoRA: Quantize Base Weights to 4-Bit, §2.2 "Double Quantization": the fp32
# block constants become "8-bit FP8" numbers.  Reading: OCP E4M3 (1 sign,
# 4 exponent bits with bias 7, 3 mantissa bits; no infinities; S.1111.111 is
# NaN; largest finite 448), round to nearest even, saturating to +-448.

E4M3_MAX = 448.0


def e4m3_decode(code) -> np.ndarray:
    """Value of each E4M3 code, by the closed form of the format."""
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    m = c & 7
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    v = np.where(e == 0, sub, normal)
    v = np.where(s == 1, -v, v)
    v = np.where((e == 15) & (m == 7), np.nan, v)
    return v.astype(F64)


def e4m3_round(v) -> np.ndarray:
    """Round to the E4M3 grid (RNE, saturate to +-448); returns the value."""
    return round_to_precision(v, 4, -6, E4M3_MAX, saturate=True)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 code (uint8) of the RNE-saturated rounding of v."""
    v = np.asarray(v, dtype=F64)
    r = e4m3_round(v)
    sign = np.signbit(v).astype(np.int64)
    a = np.abs(r)
    codes = np.zeros(v.shape, dtype=np.int64)
    nz = (a > 0) & ~np.isnan(a)
    _, e2 = np.frexp(np.where(nz, a, 1.0))
    e = e2.astype(np.int64) - 1                     # a = 1.m * 2**e
    is_normal = nz & (e >= -6)
    mant_n = np.rint((np.ldexp(np.where(nz, a, 1.0), -e) - 1.0) * 8).astype(np.int64)
    exp_field = np.where(is_normal, e + 7, 0)
    mant_s = np.rint(np.ldexp(np.where(nz, a, 0.0), 9)).astype(np.int64)   # a = m/8 * 2**-6
    mant = np.where(is_normal, mant_n, np.where(nz, mant_s, 0))
    codes = (sign << 7) | (exp_field << 3) | mant
    codes = np.where(np.isnan(v), 0x7F, codes)
    return codes.astype(np.uint8)
