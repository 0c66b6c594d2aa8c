"""FP8 E4M3 block quantisation of Q/K/V, in the oracle's own arithmetic.

The pages name FP8 attention only as prior art (cuDNN FP8 and VC-Attention FP8
attention on B200: scopeai.cc, section on the effects of each optimisation;
bpdata.com, "Kvantált attention").  The scheme here: a block is 64
consecutive tokens x all D channels of one (b, h); its scale is amax / 448
computed in fp32 (1 when amax is 0); every element x becomes the E4M3 code of
the fp32 quotient x / scale, rounded to nearest even and saturated to +-448.
Q and K are quantised after the rotary embedding, V without it.

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

from . import formats

BLOCK = 64


def block_scales(x32: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """fp32 scale per block of `block` rows of x32 [..., N, D] -> [..., ceil(N/block)]."""
    x32 = np.asarray(x32, dtype=np.float32)
    N = x32.shape[-2]
    nb = -(-N // block)
    scales = np.empty(x32.shape[:-2] + (nb,), dtype=np.float32)
    for j in range(nb):
        amax = np.abs(x32[..., j * block:(j + 1) * block, :]).max(axis=(-2, -1))
        s = (amax.astype(np.float32) / np.float32(formats.E4M3_MAX)).astype(np.float32)
        scales[..., j] = np.where(amax == 0, np.float32(1.0), s)
    return scales


def quantize(x32: np.ndarray, block: int = BLOCK):
    """E4M3 codes uint8 [..., N, D] and fp32 scales [..., ceil(N/block)] of x32."""
    x32 = np.asarray(x32, dtype=np.float32)
    scales = block_scales(x32, block)
    N = x32.shape[-2]
    per_row = np.repeat(scales, block, axis=-1)[..., :N, None]
    quot = (x32 / per_row).astype(np.float32)        # one IEEE fp32 division
    return formats.e4m3_encode(quot.astype(np.float64)), scales


def dequantize(codes: np.ndarray, scales: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """fp64 value code * scale of every element."""
    N = codes.shape[-2]
    per_row = np.repeat(np.asarray(scales, dtype=np.float64), block, axis=-1)[..., :N, None]
    return formats.e4m3_decode(codes) * per_row


def tie_count(x32: np.ndarray, scales: np.ndarray, block: int = BLOCK) -> int:
    """How many fp32 quotients x / scale land exactly halfway between two
    neighbouring E4M3 values (where round-to-nearest-even decides)."""
    x32 = np.asarray(x32, dtype=np.float32)
    N = x32.shape[-2]
    per_row = np.repeat(scales, block, axis=-1)[..., :N, None]
    quot = np.abs((x32 / per_row).astype(np.float32).astype(np.float64))
    quot = np.minimum(quot, formats.E4M3_MAX)
    down = formats.e4m3_decode(formats.e4m3_encode(quot))
    # the neighbour on the other side of the quotient
    step = np.where(quot < 2.0 ** -6, 2.0 ** -9, np.ldexp(1.0, np.frexp(np.maximum(quot, 2.0 ** -6))[1] - 4))
    other = np.where(down <= quot, down + step, down - step)
    return int(np.count_nonzero(np.abs(quot - down) == np.abs(other - quot)))
