"""Seeded synthetic workloads: sizes, positions, draws and sampled rows.  CPU only."""
import numpy as np

import workloads as W


def test_workload_sizes():
    n = {k: W.WORKLOADS[k].N for k in W.ORDER}
    assert n == {"tiny_256": 256, "t2i_512px": 1536, "t2i_1024px_cfg": 4608,
                 "t2i_2048px": 16896, "i2i_2048px": 33280}
    assert W.WORKLOADS["t2i_2048px"].flops == 4.0 * 16896 ** 2 * 128 * 24


def test_positions_layout():
    w = W.WORKLOADS["i2i_2048px"]
    p = W.positions(w)
    assert p.shape == (33280, 3) and p.dtype == np.int32
    assert not p[:512].any()                                     # text at the origin
    assert tuple(p[512]) == (0, 0, 0) and tuple(p[512 + 129]) == (0, 1, 1)
    assert tuple(p[512 + 16383]) == (0, 127, 127)
    assert tuple(p[512 + 16384]) == (1, 0, 0) and tuple(p[-1]) == (1, 127, 127)
    t = W.positions(W.WORKLOADS["tiny_256"])
    assert tuple(t[64 + 16]) == (0, 1, 0)                        # 12 x 16 grid, row-major


def test_draws_are_seeded_and_outliers_applied():
    w = W.custom(1, 2, 8, [(4, 4)], outliers=True)
    q1, k1, v1 = W.make_qkv(w, seed=0)
    q2, _, _ = W.make_qkv(w, seed=0)
    assert (q1 == q2).all()
    ch = list(W.OUTLIER_CHANNELS)
    others = [c for c in range(128) if c not in ch]
    assert q1[..., ch].float().abs().mean() > 8 * q1[..., others].float().abs().mean()
    wp = W.custom(1, 2, 8, [(4, 4)], outliers=False)
    qp, _, _ = W.make_qkv(wp, seed=0)
    # outliers are a gain on the same draw
    assert (qp[..., others] == q1[..., others]).all()


def test_sample_rows():
    small = W.WORKLOADS["tiny_256"]
    r = W.sample_rows(small)
    assert len(r) == 512
    big = W.WORKLOADS["t2i_2048px"]
    r = W.sample_rows(big)
    assert len(r) >= 4096 and len(np.unique(r, axis=0)) == len(r)
    rows = {tuple(x) for x in r}
    for b, h in ((0, 0), (0, 23)):
        for n in (0, 511, 512, 16895):
            assert (b, h, n) in rows
    assert np.array_equal(r, W.sample_rows(big))
