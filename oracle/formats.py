"""Number formats used by the oracle: round-to-nearest-even into bf16, fp16,
fp32 (and the two-term fp16 split of an fp32 value) and into OCP FP8 E4M3 ("e4m3fn": bias 7, largest finite 448, no infinities, NaN is
S.1111.111), written from the formats' definitions in fp64 arithmetic.

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def _round_nearest_even(x, sig_bits: int, min_exp: int):
    """Round fp64 values to a binary format with `sig_bits` significand bits
    (implicit bit included) whose smallest normal exponent is `min_exp`.

    Below 2**min_exp the spacing stays 2**(min_exp - sig_bits + 1) (gradual
    underflow).  Ties go to the even neighbour (numpy.rint).  Range overflow is
    left to the caller.  Scaling by a power of two is exact in fp64, so the only
    rounding here is the single rint.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    _, e = np.frexp(ax)                       # ax = f * 2**e, 0.5 <= f < 1
    lead = np.maximum(e - 1, min_exp)         # exponent of the leading bit
    spacing = np.ldexp(1.0, lead - (sig_bits - 1))
    r = np.rint(ax / spacing) * spacing
    return np.copysign(r, x)


def round_bf16(x):
    """Nearest-even bf16 value of fp64 `x`, returned as fp64.

    bf16: 8 significand bits, exponent range of IEEE binary32 (smallest normal
    2**-126); magnitudes at or above the overflow threshold become inf.
    """
    r = _round_nearest_even(x, 8, -126)
    bf16_max = (2.0 - 2.0 ** -7) * 2.0 ** 127
    overflow = np.abs(r) > bf16_max
    return np.where(overflow, np.copysign(np.inf, r), r)


def round_fp16(x):
    """Nearest-even IEEE binary16 value of fp64 `x` (11 significand bits,
    smallest normal 2**-14, largest finite 65504), returned as fp64."""
    r = _round_nearest_even(x, 11, -14)
    overflow = np.abs(r) > 65504.0
    return np.where(overflow, np.copysign(np.inf, r), r)


def round_fp32(x):
    """Nearest-even IEEE binary32 value of fp64 `x` (24 significand bits,
    smallest normal 2**-126), returned as fp64; overflow becomes inf."""
    r = _round_nearest_even(x, 24, -126)
    fp32_max = (2.0 - 2.0 ** -23) * 2.0 ** 127
    return np.where(np.abs(r) > fp32_max, np.copysign(np.inf, r), r)


def split_fp16(r):
    """Two-term fp16 representation of fp32 values r (given as fp64):
    hi = the fp16 nearest r, lo = the fp16 nearest r - hi.  The difference is
    formed in fp64, where it is exact.  hi + lo is within half an fp16 ulp of
    lo of r: 2**-22 |r| relative, 2**-25 absolute where lo is subnormal.
    This is the operand format of the compensated (split) q k^T."""
    r = np.asarray(r, dtype=np.float64)
    hi = round_fp16(r)
    lo = round_fp16(r - hi)
    return hi, lo


def e4m3_decode(codes):
    """Value of each E4M3 code (uint8) as fp64; 0x7F / 0xFF decode to NaN.

    Field layout: sign bit 7, exponent bits 6..3 (bias 7), mantissa bits 2..0.
    Exponent field 0 encodes subnormals m * 2**-9.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    ef = (c >> 3) & 0xF
    mf = c & 0x7
    normal = (1.0 + mf / 8.0) * np.ldexp(1.0, ef - 7)
    sub = mf * 2.0 ** -9
    val = np.where(ef == 0, sub, normal)
    val = np.where((ef == 15) & (mf == 7), np.nan, val)
    return sign * val


def e4m3_encode(x):
    """E4M3 code (uint8) of fp64 `x`: round to nearest even, saturating to
    +-448 (the "satfinite" conversion); NaN maps to 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    nan = np.isnan(x)
    r = _round_nearest_even(np.where(nan, 0.0, x), 4, -6)
    r = np.clip(r, -E4M3_MAX, E4M3_MAX)
    sign = (np.signbit(r)).astype(np.int64) << 7
    ar = np.abs(r)
    code = np.zeros(ar.shape, dtype=np.int64)
    sub = ar < 2.0 ** -6
    code = np.where(sub, np.rint(ar / 2.0 ** -9).astype(np.int64), code)
    _, e = np.frexp(np.where(sub, 1.0, ar))
    lead = e - 1                                        # ar = 1.m * 2**lead
    mant = np.rint((np.where(sub, 1.0, ar) / np.ldexp(1.0, lead) - 1.0) * 8.0).astype(np.int64)
    normal_code = ((lead + 7) << 3) | mant
    code = np.where(sub, code, normal_code)
    code = np.where(nan, 0x7F, code | sign)
    return code.astype(np.uint8)
