"""The QKV projection that feeds the joint attention, in fp64, and the FP8
operands made from it.

Inside a DiT block the attention's q, k and v come from one linear layer
over the hidden states of the joint token sequence (text and image tokens
alike):

    y[b, n, o] = sum_c x[b, n, c] w[o, c]  (+ bias[o]),   o = s H D + h D + d

with s = 0, 1, 2 for q, k, v, head h and channel d, so that q[b, h, n, d] =
y[b, n, h D + d] and so on.  The pages put GEMMs with epilogue fusion among
the optimisations of FLUX 3 Klein on B200 (bpdata.com "FLUX 3 Image Klein
optimalizálása", section on what the optimisation includes); the epilogue
fused here is the rotary embedding of q and k and the block quantisation of
the FP8 attention operands (oracle.fp8).

Written as the definition: one fp64 matrix product per batch item (a library
primitive; every product of bf16 values is exact in fp64 and the sum is
rounded there), the bias added, the columns regrouped per head.  Test
infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

from . import attention, fp8, rope


def project(x, w, bias=None, H: int = 24, D: int = 128):
    """(q, k, v), each fp64 [B, H, N, D], of x [B, N, C] and w [3 H D, C]."""
    x = attention.to_f64(x)
    w = attention.to_f64(w)
    y = np.einsum("bnc,oc->bno", x, w)
    if bias is not None:
        y = y + attention.to_f64(bias)[None, None, :]
    B, N, _ = y.shape
    y = y.reshape(B, N, 3, H, D).transpose(2, 0, 3, 1, 4)          # [3, B, H, N, D]
    return y[0], y[1], y[2]


def magnitude(x, w, H: int = 24, D: int = 128):
    """sum_c |x[b, n, c] w[o, c]| per output element, regrouped like project():
    the scale of the rounding error of any summation order of the products."""
    y = np.einsum("bnc,oc->bno", np.abs(attention.to_f64(x)), np.abs(attention.to_f64(w)))
    B, N, _ = y.shape
    y = y.reshape(B, N, 3, H, D).transpose(2, 0, 3, 1, 4)
    return y[0], y[1], y[2]


def rotated_fp32(y, pos):
    """The rotated projection of q or k as the FP8 quantiser takes it: each
    pair turned with the fp32 table entries in fp64 (both products of fp32
    values are exact there, the sum rounded once) and rounded to fp32."""
    from . import formats
    c, s = rope.table_fp32(pos)
    return formats.round_fp32(rope.rotate_with_table(y, c, s))
