"""Seeded synthetic inputs for the joint text+image attention workloads.

This module is shared by the fp64 oracle's tests and by the CUDA path's tests
and benchmark.  It holds no arithmetic of the method itself (no rotary
embedding, no softmax, no quantisation): only the workload table, the token
positions, the seeded random Q/K/V draws and the seeded choice of sampled
query rows.

Workloads (FLUX-style DiT joint attention, head dim 128 throughout).  The
joint sequence is [text | target image | (reference image)], the order in
which the FLUX 3 Klein DiT handles its text, noisy-target and optional
reference-image inputs before merging them in a shared attention layer
(bpdata.com "FLUX 3 Image Klein optimalizálása", section "Modellezés és
pipeline jellemzők").  Image resolutions 512/1024/2048 px, the CFG batch of
two and the image-to-image case follow the workloads those pages measure
(wavespeed.ai FLUX.1-dev results table; scopeai.cc test-conditions section).
Head count, head dim, text length, latent grids, rotary axis split and the
outlier-channel pattern are not on the pages; they are fixed here.
"""
from __future__ import annotations

import dataclasses
from typing import List, Tuple

import numpy as np
import torch

HEAD_DIM = 128
ROPE_AXES = (16, 56, 56)          # channels per rotary axis (t, h, w)
ROPE_THETA = 10000.0
OUTLIER_CHANNELS = (3, 40, 77, 110)   # one in t, one in h, two in w
OUTLIER_GAIN = 16.0
SAMPLE_ROWS = 4096
FULL_ROWS_LIMIT = 4096


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    n_txt: int
    grids: Tuple[Tuple[int, int], ...]   # (rows, cols) per image, in sequence order
    outliers: bool
    D: int = HEAD_DIM

    @property
    def n_img(self) -> int:
        return sum(r * c for r, c in self.grids)

    @property
    def N(self) -> int:
        return self.n_txt + self.n_img

    @property
    def flops(self) -> float:
        """Dense attention work: 2*N*N*D for Q.K^T plus 2*N*N*D for P.V, per (b, h)."""
        return 4.0 * self.N * self.N * self.D * self.H * self.B

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "D": self.D,
                "n_txt": self.n_txt, "n_img": self.n_img, "N": self.N,
                "grids": [list(g) for g in self.grids],
                "inputs": "N(0,1) bf16" + (" with channels %s x%g" % (
                    list(OUTLIER_CHANNELS), OUTLIER_GAIN) if self.outliers else "")}


WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_256", B=1, H=2, n_txt=64, grids=((12, 16),), outliers=False),
        Workload("t2i_512px", B=1, H=24, n_txt=512, grids=((32, 32),), outliers=False),
        Workload("t2i_1024px_cfg", B=2, H=24, n_txt=512, grids=((64, 64),), outliers=False),
        Workload("t2i_2048px", B=1, H=24, n_txt=512, grids=((128, 128),), outliers=True),
        Workload("i2i_2048px", B=1, H=24, n_txt=512, grids=((128, 128), (128, 128)), outliers=True),
    ]
}
ORDER = ["tiny_256", "t2i_512px", "t2i_1024px_cfg", "t2i_2048px", "i2i_2048px"]


def custom(B: int, H: int, n_txt: int, grids, outliers: bool = False, name: str = "custom") -> Workload:
    return Workload(name, B=B, H=H, n_txt=n_txt, grids=tuple(tuple(g) for g in grids), outliers=outliers)


def positions(w: Workload) -> np.ndarray:
    """Integer (t, h, w) position of every token, int32 [N, 3].

    Text tokens sit at (0, 0, 0).  Image g (0 = target, 1 = reference) places
    its latent pixel (row, col) at (g, row, col), row-major.
    """
    out = np.zeros((w.N, 3), dtype=np.int32)
    off = w.n_txt
    for g, (rows, cols) in enumerate(w.grids):
        r, c = np.meshgrid(np.arange(rows), np.arange(cols), indexing="ij")
        n = rows * cols
        out[off:off + n, 0] = g
        out[off:off + n, 1] = r.reshape(-1)
        out[off:off + n, 2] = c.reshape(-1)
        off += n
    return out


def make_qkv(w: Workload, seed: int = 0):
    """Q, K, V as bf16 CPU tensors [B, H, N, D].

    Drawn as float32 N(0, 1) from one torch CPU generator seeded with `seed`, in
    the order Q, K, V.  For outlier workloads the channels OUTLIER_CHANNELS are
    multiplied by OUTLIER_GAIN in all three tensors, for every token, batch and
    head, before the round-to-nearest-even cast to bf16.
    """
    g = torch.Generator(device="cpu").manual_seed(seed)
    shape = (w.B, w.H, w.N, w.D)
    out = []
    for _ in range(3):
        x = torch.randn(shape, generator=g, dtype=torch.float32)
        if w.outliers:
            x[..., list(OUTLIER_CHANNELS)] *= OUTLIER_GAIN
        out.append(x.to(torch.bfloat16))
    return tuple(out)


def sample_rows(w: Workload, seed: int = 1, count: int = SAMPLE_ROWS) -> np.ndarray:
    """Seeded (b, h, n) query rows to check, int64 [R, 3], sorted.

    Every row when B*H*N <= FULL_ROWS_LIMIT.  Otherwise the first `count` of a
    seeded permutation of all B*H*N rows, plus fixed edge rows: the first and
    last text row, the first image row and the last row, of (b=0, h=0) and of
    (b=B-1, h=H-1), and the last row of the 128-row tile that holds
    n = N // 2 in every head.
    """
    total = w.B * w.H * w.N
    if total <= FULL_ROWS_LIMIT:
        flat = np.arange(total, dtype=np.int64)
    else:
        g = torch.Generator().manual_seed(seed)
        flat = torch.randperm(total, generator=g)[:count].numpy().astype(np.int64)
        extra = []
        for b, h in ((0, 0), (w.B - 1, w.H - 1)):
            for n in (0, max(w.n_txt - 1, 0), min(w.n_txt, w.N - 1), w.N - 1):
                extra.append((b * w.H + h) * w.N + n)
        mid_tile_end = min((w.N // 2) // 128 * 128 + 127, w.N - 1)
        for b in range(w.B):
            for h in range(w.H):
                extra.append((b * w.H + h) * w.N + mid_tile_end)
        flat = np.unique(np.concatenate([flat, np.asarray(extra, dtype=np.int64)]))
    b = flat // (w.H * w.N)
    h = (flat // w.N) % w.H
    n = flat % w.N
    return np.stack([b, h, n], axis=1)


def group_rows(rows: np.ndarray) -> List[Tuple[int, int, np.ndarray]]:
    """Split sampled rows into (b, h, n-array) groups, in (b, h) order."""
    out = []
    keys = rows[:, 0] * 1_000_000 + rows[:, 1]
    for key in np.unique(keys):
        sel = rows[keys == key]
        out.append((int(sel[0, 0]), int(sel[0, 1]), sel[:, 2].copy()))
    return out
