"""Combination of partial attention results over disjoint key sets.

Context parallelism (wavespeed.ai "Beschleunigung der FLUX.1-dev
Bildgenerierung", context-parallel + First Block Cache section) splits the
sequence over GPUs; each part attends to its own slice of keys and returns a
partial output O_r with its log-sum-exp lse_r.  The exact result over the
union of the slices is

    lse = log sum_r exp(lse_r)
    O   = sum_r exp(lse_r - lse) O_r

A part whose key slice is empty has sum exp = 0, so lse_r = -inf: its weight
is exp(-inf) = 0 and its O_r (undefined: 0/0) is ignored.  When every part is
empty the union is empty too: lse = -inf and O is taken as 0.

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np


def merge(outs, lses):
    """outs: sequence of [R, D] partial outputs; lses: matching [R] log-sum-exps."""
    lses = np.stack([np.asarray(l, dtype=np.float64) for l in lses])       # [P, R]
    outs = np.stack([np.asarray(o, dtype=np.float64) for o in outs])       # [P, R, D]
    m = lses.max(axis=0)
    empty = np.isneginf(m)                                   # no part has a key
    m_ref = np.where(empty, 0.0, m)
    w = np.exp(lses - m_ref[None, :])                        # 0 for empty parts
    total = w.sum(axis=0)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m_ref + np.log(np.where(empty, 1.0, total)))
    terms = np.where(w[:, :, None] > 0, w[:, :, None] * outs, 0.0)     # an empty part's O is not read
    out = terms.sum(axis=0) / np.where(empty, 1.0, total)[:, None]
    return out, lse
