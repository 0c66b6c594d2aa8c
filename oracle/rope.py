"""Three-axis rotary position embedding (t, h, w), in fp64.

The pages describe the FLUX DiT only as processing text, target and reference
image inputs jointly in one attention layer (bpdata.com "FLUX 3 Image Klein
optimalizálása", section "Modellezés és pipeline jellemzők"); they give no
rotary convention.  The one used here is the plain per-axis RoFormer form:

* the head dimension is split into consecutive axis slices of widths
  axes = (d_t, d_h, d_w), by default (16, 56, 56) at channel offsets 0, 16, 72;
* inside axis slice a, channel pair i (channels o_a + 2i and o_a + 2i + 1)
  turns by the angle  phi = pos_a * theta ** (-2 i / d_a),  theta = 10000;
* the pair (x, y) becomes (x cos phi - y sin phi, x sin phi + y cos phi).

Pair columns are laid out in channel order: column j of an angle table is the
pair of channels (2j, 2j + 1).

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

DEFAULT_AXES = (16, 56, 56)
DEFAULT_THETA = 10000.0


def frequencies(axes=DEFAULT_AXES, theta: float = DEFAULT_THETA):
    """(axis index, omega) for every channel pair, in channel order."""
    axis_of_pair = []
    omega = []
    for a, d in enumerate(axes):
        if d % 2:
            raise ValueError("rotary axis widths must be even")
        for i in range(d // 2):
            axis_of_pair.append(a)
            omega.append(theta ** (-2.0 * i / d))
    return np.asarray(axis_of_pair, dtype=np.int64), np.asarray(omega, dtype=np.float64)


def angles(pos, axes=DEFAULT_AXES, theta: float = DEFAULT_THETA):
    """Rotation angle of every (token, channel pair): fp64 [N, sum(axes)/2]."""
    pos = np.asarray(pos)
    axis_of_pair, omega = frequencies(axes, theta)
    return pos[:, axis_of_pair].astype(np.float64) * omega[None, :]


def table(pos, axes=DEFAULT_AXES, theta: float = DEFAULT_THETA):
    """cos and sin of `angles`, each fp64 [N, sum(axes)/2]."""
    phi = angles(pos, axes, theta)
    return np.cos(phi), np.sin(phi)


def table_fp32(pos, axes=DEFAULT_AXES, theta: float = DEFAULT_THETA):
    """The table as the library stores it: each fp64 entry rounded to the
    nearest fp32 value (returned as fp64)."""
    c, s = table(pos, axes, theta)
    return c.astype(np.float32).astype(np.float64), s.astype(np.float32).astype(np.float64)


def rotate(x, phi):
    """Apply the rotation of angle table `phi` [N, D/2] to x [..., N, D] (fp64)."""
    return rotate_with_table(x, np.cos(phi), np.sin(phi))


def rotate_with_table(x, c, s):
    """Apply the rotation whose cos / sin entries are c, s [N, D/2] to x [..., N, D] (fp64)."""
    x = np.asarray(x, dtype=np.float64)
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def rotate_split(x, c, s):
    """Operands of the compensated (split) q k^T: the rotation of x [..., N, D]
    with the table entries c, s [N, D/2], each component evaluated in fp64
    (both products exact for bf16 x and fp32 entries, the sum rounded once)
    and rounded to fp32, then split into fp16 hi + lo (formats.split_fp16).
    Returns (hi, lo) as fp64 arrays of x's shape."""
    from . import formats
    r = formats.round_fp32(rotate_with_table(x, c, s))
    return formats.split_fp16(r)
