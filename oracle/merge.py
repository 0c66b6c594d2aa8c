"""Combination of partial attention results over disjoint key sets.

Context parallelism (wavespeed.ai "Beschleunigung der FLUX.1-dev
Bildgenerierung", context-parallel + First Block Cache section) splits the
sequence over GPUs; each part attends to its own slice of keys and returns a
partial output O_r with its log-sum-exp lse_r.  The exact result over the
union of the slices is

    lse = log sum_r exp(lse_r)
    O   = sum_r exp(lse_r - lse) O_r

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np


def merge(outs, lses):
    """outs: sequence of [R, D] partial outputs; lses: matching [R] log-sum-exps."""
    lses = np.stack([np.asarray(l, dtype=np.float64) for l in lses])       # [P, R]
    outs = np.stack([np.asarray(o, dtype=np.float64) for o in outs])       # [P, R, D]
    m = lses.max(axis=0)
    w = np.exp(lses - m[None, :])
    total = w.sum(axis=0)
    lse = m + np.log(total)
    out = (w[:, :, None] * outs).sum(axis=0) / total[:, None]
    return out, lse
