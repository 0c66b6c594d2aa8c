"""Bidirectional joint text+image attention with rotary Q/K, in fp64.

What is computed, for every batch item b and head h separately (the heads of
a DiT block attend independently; text and image tokens of one item form one
sequence that every token attends to in full, which is the "shared attention
layer" of bpdata.com "FLUX 3 Image Klein optimalizálása", section
"Modellezés és pipeline jellemzők"):

    q~_n = R(pos_n) q_n,   k~_m = R(pos_m) k_m          (oracle.rope)
    s_nm = (q~_n . k~_m) * scale,   scale = 1 / sqrt(D)
    O_n  = sum_m softmax_m(s_n.) v_m
    LSE_n = log sum_m exp(s_nm)          (natural log, scaled-logit units)

written as the definition: a full row of logits, its maximum subtracted
before exp (which changes nothing mathematically), the exponentials summed,
and one weighted sum of V.  No tiling, streaming or rescaling.

Two optional rounding points model the formats the library's interface fixes
for intermediate values, with exact arithmetic in between:
* `table_fp32=True` rotates with the cos / sin table entries rounded to fp32
  (the table format the attention call takes);
* `round_rotated="bf16"` rounds the exactly rotated q~ and k~ to the nearest
  bf16 (ties to even): the operand precision of a bf16 tensor-core product.
Everything else stays fp64.

With `kv_mask` the sum runs over the keys of the allowed (query block, key
tile) pairs only: the block-sparse form that skips whole tiles (a generic
stand-in for the sparse attention the pages name as prior art: scopeai.cc,
section on each optimisation's effect; bpdata.com, section on the reference
kernels).

Test infrastructure only (see oracle/__init__.py).
"""
from __future__ import annotations

import numpy as np

from . import formats, rope


def to_f64(x) -> np.ndarray:
    """Exact fp64 copy of a numpy array or a (CPU) torch tensor of any float dtype."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attention_rows(q_rows, k, v, scale, allowed=None):
    """softmax(q_rows k^T * scale) v for one (b, h): returns O [R, D], LSE [R].

    allowed: optional bool [R, N], the keys each row attends to; the others
    are left out of the softmax (their logits taken as -inf).  A row with no
    key has an empty sum: O = 0 and LSE = -inf.
    """
    s = (q_rows @ k.T) * scale
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
        empty = ~allowed.any(axis=1)
        s[empty] = 0.0                       # placeholder logits, result replaced below
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    if allowed is not None:
        e = np.where(allowed | empty[:, None], e, 0.0)
    l = e.sum(axis=1, keepdims=True)
    out = (e @ v) / l
    lse = m[:, 0] + np.log(l[:, 0])
    if allowed is not None:
        out[empty] = 0.0
        lse[empty] = -np.inf
    return out, lse


def probabilities(q_rows, k, scale):
    """Full attention probability rows softmax(q_rows k^T * scale) [R, N]."""
    s = (q_rows @ k.T) * scale
    e = np.exp(s - s.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def _round(x, how):
    if how is None:
        return x
    if how == "bf16":
        return formats.round_bf16(x)
    if how == "fp16":
        return formats.round_fp16(x)
    raise ValueError(how)


def joint_attention(q, k, v, pos=None, rows=None, axes=rope.DEFAULT_AXES,
                    theta: float = rope.DEFAULT_THETA, scale=None, round_rotated=None, table_fp32=False,
                    kv_mask=None, q_block: int = 512, kv_block: int = 128):
    """Oracle output for tensors q, k, v [B, H, N, D].

    pos:  int [N, 3] token positions (t, h, w) or None for no rotary embedding.
    rows: int [R, 3] (b, h, n) query rows to evaluate, or None for all rows.
    kv_mask: optional [B, H, ceil(N / q_block), ceil(N / kv_block)] array:
          query n of (b, h) attends to key m only where
          kv_mask[b, h, n // q_block, m // kv_block] is nonzero (block-sparse
          attention; the selection rule is the caller's).
    Returns (O [R, D], LSE [R]) in fp64, in the order of `rows` (row-major
    (b, h, n) order when rows is None).
    """
    B, H, N, D = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    if rows is None:
        b, h, n = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
        rows = np.stack([b.reshape(-1), h.reshape(-1), n.reshape(-1)], axis=1)
    rows = np.asarray(rows, dtype=np.int64)
    cs = None
    if pos is not None:
        cs = rope.table_fp32(pos, axes, theta) if table_fp32 else rope.table(pos, axes, theta)
    out = np.empty((len(rows), D), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    keys = rows[:, 0] * (H + 1) + rows[:, 1]
    for key in np.unique(keys):
        idx = np.nonzero(keys == key)[0]
        bb, hh = int(rows[idx[0], 0]), int(rows[idx[0], 1])
        kk = to_f64(k[bb, hh])
        vv = to_f64(v[bb, hh])
        qq = to_f64(q[bb, hh][rows[idx, 2]])
        if cs is not None:
            kk = rope.rotate_with_table(kk, cs[0], cs[1])
            qq = rope.rotate_with_table(qq, cs[0][rows[idx, 2]], cs[1][rows[idx, 2]])
        kk = _round(kk, round_rotated)
        qq = _round(qq, round_rotated)
        allowed = None
        if kv_mask is not None:
            blocks = np.asarray(kv_mask)[bb, hh] != 0                       # [n_qblk, n_kvblk]
            allowed = blocks[rows[idx, 2] // q_block][:, np.arange(N) // kv_block]
        o, l = attention_rows(qq, kk, vv, scale, allowed)
        out[idx] = o
        lse[idx] = l
    return out, lse
