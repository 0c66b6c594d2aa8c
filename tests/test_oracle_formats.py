"""Pins for oracle.formats and oracle.fp8: the OCP E4M3 definition's landmark
codes, exhaustive round trips, tie rules, and library conversions (torch's
fp32->bf16 / fp16 / float8_e4m3fn casts) as independent checks.  CPU only."""
import numpy as np
import pytest
import torch

from oracle import formats, fp8


def _torch_round(x32, dtype):
    return torch.from_numpy(np.asarray(x32, dtype=np.float32)).to(dtype).to(torch.float64).numpy()


def test_round_bf16_matches_library_cast_on_fp32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    assert np.array_equal(formats.round_bf16(x.astype(np.float64)), _torch_round(x, torch.bfloat16))


def test_round_bf16_ties_go_to_even():
    one = 1.0
    ulp = 2.0 ** -7
    # halfway between 1 and 1+ulp -> 1 (even); halfway between 1+ulp and 1+2ulp -> 1+2ulp
    assert formats.round_bf16(one + ulp / 2) == one
    assert formats.round_bf16(one + 1.5 * ulp) == one + 2 * ulp
    assert formats.round_bf16(-(one + 1.5 * ulp)) == -(one + 2 * ulp)
    # just above halfway rounds up
    assert formats.round_bf16(one + ulp / 2 + 2.0 ** -40) == one + ulp
    # carry into the next binade
    assert formats.round_bf16(2.0 - 2.0 ** -9) == 2.0


def test_round_fp16_matches_library_cast():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(200000) * np.exp(rng.uniform(-12, 10, 200000))).astype(np.float32)
    assert np.array_equal(formats.round_fp16(x.astype(np.float64)), _torch_round(x, torch.float16))
    assert formats.round_fp16(70000.0) == np.inf


def test_e4m3_landmark_codes():
    d = formats.e4m3_decode
    assert d(0x7E) == 448.0           # largest finite: 1.75 * 2^8
    assert d(0xFE) == -448.0
    assert d(0x38) == 1.0             # exponent field 7 = bias
    assert d(0x08) == 2.0 ** -6       # smallest normal
    assert d(0x07) == 7 * 2.0 ** -9   # largest subnormal
    assert d(0x01) == 2.0 ** -9       # smallest subnormal
    assert d(0x00) == 0.0
    assert np.isnan(d(0x7F)) and np.isnan(d(0xFF))
    assert d(0x77) == 240.0           # 1.875 * 2^7
    assert d(0x3C) == 1.5


def test_e4m3_exhaustive_round_trip_and_ordering():
    codes = np.arange(256, dtype=np.uint8)
    vals = formats.e4m3_decode(codes)
    finite = ~np.isnan(vals)
    back = formats.e4m3_encode(vals[finite])
    # +0 and -0 both decode to 0; the encoder keeps the sign bit
    assert np.array_equal(back, codes[finite])
    pos = np.sort(vals[finite & (vals >= 0)])
    assert len(np.unique(pos)) == 127 and pos[-1] == 448.0


def test_e4m3_midpoints_round_to_even_and_saturate():
    vals = np.sort(np.unique(formats.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))))
    mids = (vals[:-1] + vals[1:]) / 2
    enc = formats.e4m3_encode(mids)
    lo = formats.e4m3_encode(vals[:-1])
    hi = formats.e4m3_encode(vals[1:])
    expect = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(enc, expect)
    assert formats.e4m3_encode(500.0) == 0x7E and formats.e4m3_encode(-1e9) == 0xFE
    assert formats.e4m3_encode(464.0) == 0x7E      # the would-be midpoint to 480 saturates
    assert formats.e4m3_encode(np.nan) == 0x7F


def test_e4m3_encode_matches_library_cast():
    rng = np.random.default_rng(2)
    x = (rng.uniform(-448, 448, 100000) * np.exp(rng.uniform(-14, 0, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(formats.e4m3_encode(x.astype(np.float64)), ref)


def test_block_quantisation_properties():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((2, 3, 200, 128)) * 4).astype(np.float32)
    x[0, 1, 64:128] = 0.0                      # an all-zero block
    codes, scales = fp8.quantize(x)
    assert codes.dtype == np.uint8 and scales.shape == (2, 3, 4)
    assert scales[0, 1, 1] == 1.0 and not codes[0, 1, 64:128].any()
    # the largest magnitude of every non-zero block lands on +-448
    for b in range(2):
        for h in range(3):
            for j in range(4):
                blk = x[b, h, j * 64:(j + 1) * 64]
                if np.abs(blk).max() == 0:
                    continue
                i = np.unravel_index(np.abs(blk).argmax(), blk.shape)
                assert formats.e4m3_decode(codes[b, h, j * 64 + i[0], i[1]]) == np.sign(blk[i]) * 448.0
    # rounding error of every element stays within half a code step
    deq = fp8.dequantize(codes, scales)
    per_row = np.repeat(scales, 64, axis=-1)[..., :200, None].astype(np.float64)
    rel = np.abs(x / per_row)
    half_step = np.where(rel < 2.0 ** -6, 2.0 ** -10, np.ldexp(1.0, np.frexp(np.maximum(rel, 2.0 ** -6))[1] - 5))
    assert np.all(np.abs(deq - x) <= half_step * per_row * (1 + 1e-6) + 1e-30)


def test_tie_count_finds_constructed_ties():
    x = np.zeros((1, 64, 4), dtype=np.float32)
    x[0, 0, 0] = 448.0            # scale 1
    x[0, 1, 0] = 1.0625           # halfway between 1.0 and 1.125
    x[0, 2, 0] = 1.05             # not a tie
    scales = fp8.block_scales(x)
    assert scales[0, 0] == 1.0
    assert fp8.tie_count(x, scales) == 1


def test_round_fp32_matches_library_cast_and_ties_to_even():
    rng = np.random.default_rng(5)
    x = rng.standard_normal(200000) * np.exp(rng.uniform(-95, 85, 200000))
    assert np.array_equal(formats.round_fp32(x), x.astype(np.float32).astype(np.float64))
    ulp = 2.0 ** -23
    assert formats.round_fp32(1.0 + ulp / 2) == 1.0
    assert formats.round_fp32(1.0 + 1.5 * ulp) == 1.0 + 2 * ulp
    assert formats.round_fp32(2.0 ** -140 * 1.25) == np.float64(np.float32(2.0 ** -140 * 1.25))   # subnormal
    assert formats.round_fp32(4.0e38) == np.inf


def test_split_fp16_terms():
    rng = np.random.default_rng(6)
    r = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 10, 100000))).astype(np.float32).astype(np.float64)
    hi, lo = formats.split_fp16(r)
    # hi is the library's fp16 cast of r; lo the cast of the exact remainder
    assert np.array_equal(hi, _torch_round(r, torch.float16))
    assert np.array_equal(lo, _torch_round(r - hi, torch.float16))
    # hi + lo carries r to 2^-22 relative (2^-25 absolute once lo is subnormal)
    assert np.all(np.abs(hi + lo - r) <= np.maximum(2.0 ** -22 * np.abs(r), 2.0 ** -25))
    # the remainder is at most half an fp16 ulp of hi
    assert np.all(np.abs(r - hi) <= np.ldexp(1.0, np.frexp(np.abs(hi))[1] - 12) + 2.0 ** -25)
    # worked cases: exactly representable, a remainder one fp16 ulp below, a subnormal remainder
    assert formats.split_fp16(0.75) == (0.75, 0.0)
    assert formats.split_fp16(1.0 + 2.0 ** -15) == (1.0, 2.0 ** -15)
    assert formats.split_fp16(1.0 + 2.0 ** -21) == (1.0, 2.0 ** -21)
    # remainder 1.5 * 2^-24 lies halfway between the fp16 subnormals 2^-24 and 2^-23: the even one is taken
    h, l = formats.split_fp16(2.0 ** -12 + 1.5 * 2.0 ** -24)
    assert h == 2.0 ** -12 and l == 2.0 ** -23
    assert formats.split_fp16(-3.0 - 2.0 ** -14) == (-3.0, -(2.0 ** -14))
