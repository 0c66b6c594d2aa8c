"""Pins of oracle.projection: the QKV projection against exact rational
arithmetic on tiny inputs, its regrouping of output features into q, k, v
heads, and its error-scale companion.  CPU only."""
from fractions import Fraction

import numpy as np

from oracle import formats, projection


def _bf16(rng, shape, scale=1.0):
    return formats.round_bf16(rng.standard_normal(shape) * scale)


def test_project_matches_exact_rational_sums():
    rng = np.random.default_rng(11)
    B, N, C, H, D = 2, 3, 5, 2, 4
    x = _bf16(rng, (B, N, C))
    w = _bf16(rng, (3 * H * D, C))
    bias = _bf16(rng, (3 * H * D,))
    q, k, v = projection.project(x, w, bias, H=H, D=D)
    for s, y in enumerate((q, k, v)):
        for b in range(B):
            for h in range(H):
                for n in range(N):
                    for d in range(D):
                        o = s * H * D + h * D + d
                        exact = sum(Fraction(float(x[b, n, c])) * Fraction(float(w[o, c])) for c in range(C))
                        exact += Fraction(float(bias[o]))
                        assert abs(Fraction(float(y[b, h, n, d])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + \
                            Fraction(1, 2 ** 80)


def test_project_regroups_features_into_q_k_v_heads():
    """A weight that copies input channel c(o) into feature o: q[b, h, n, d]
    must be x[b, n, c(s H D + h D + d)]."""
    rng = np.random.default_rng(12)
    B, N, H, D = 1, 4, 3, 2
    C = 3 * H * D
    x = _bf16(rng, (B, N, C))
    perm = rng.permutation(C)
    w = np.zeros((C, C))
    w[np.arange(C), perm] = 1.0
    q, k, v = projection.project(x, w, H=H, D=D)
    for s, y in enumerate((q, k, v)):
        for h in range(H):
            for d in range(D):
                assert np.array_equal(y[0, h, :, d], x[0, :, perm[s * H * D + h * D + d]])


def test_magnitude_bounds_the_projection():
    rng = np.random.default_rng(13)
    x = _bf16(rng, (1, 6, 16))
    w = _bf16(rng, (3 * 2 * 4, 16))
    y = projection.project(x, w, H=2, D=4)
    m = projection.magnitude(x, w, H=2, D=4)
    for a, b in zip(y, m):
        assert np.all(np.abs(a) <= b + 1e-12) and np.all(b >= 0)
    # equality for non-negative operands
    ya = projection.project(np.abs(x), np.abs(w), H=2, D=4)
    for a, b in zip(ya, m):
        assert np.allclose(a, b, rtol=1e-14, atol=0)
