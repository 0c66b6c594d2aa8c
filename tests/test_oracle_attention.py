"""Pins for oracle.attention and oracle.rope: 50-digit brute force, a library
attention routine, closed forms and invariants.  CPU only."""
import math

import mpmath
import numpy as np
import pytest
import torch

from oracle import attention, merge, rope


def _rand_case(rng, N, D, axes, pos_hi=6):
    q = rng.standard_normal((N, D))
    k = rng.standard_normal((N, D))
    v = rng.standard_normal((N, D))
    pos = rng.integers(0, pos_hi, size=(N, 3)).astype(np.int32)
    return q, k, v, pos


def _mp_attention(q, k, v, pos, axes, theta):
    """Brute force at 50 digits with the rotation written as complex products:
    channel pair (x, y) is the complex number x + iy, turned by exp(i*phi)."""
    mpmath.mp.dps = 50
    N, D = q.shape

    def rot(vec, p):
        out = []
        off = 0
        for a, d in enumerate(axes):
            for i in range(d // 2):
                w = mpmath.power(mpmath.mpf(theta), -mpmath.mpf(2 * i) / d)
                z = mpmath.mpc(vec[off + 2 * i], vec[off + 2 * i + 1]) * mpmath.expj(int(p[a]) * w)
                out += [z.real, z.imag]
            off += d
        return out

    qs = [rot([mpmath.mpf(float(x)) for x in q[n]], pos[n]) for n in range(N)]
    ks = [rot([mpmath.mpf(float(x)) for x in k[n]], pos[n]) for n in range(N)]
    scale = 1 / mpmath.sqrt(D)
    O = np.zeros((N, D))
    L = np.zeros(N)
    for n in range(N):
        logits = [scale * mpmath.fsum(qs[n][c] * ks[m][c] for c in range(D)) for m in range(N)]
        ws = [mpmath.exp(s) for s in logits]
        tot = mpmath.fsum(ws)
        for c in range(D):
            O[n, c] = float(mpmath.fsum(ws[m] * mpmath.mpf(float(v[m, c])) for m in range(N)) / tot)
        L[n] = float(mpmath.log(tot))
    return O, L


@pytest.mark.parametrize("N,axes,seed", [(5, (2, 2, 4), 0), (12, (2, 2, 4), 1), (16, (4, 6, 6), 2), (9, (4, 6, 6), 3)])
def test_brute_force_50_digits(N, axes, seed):
    rng = np.random.default_rng(seed)
    D = sum(axes)
    q, k, v, pos = _rand_case(rng, N, D, axes)
    O_mp, L_mp = _mp_attention(q, k, v, pos, axes, 10000.0)
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos, axes=axes)
    assert np.max(np.abs(O - O_mp)) < 1e-13
    assert np.max(np.abs(L - L_mp)) < 1e-13


@pytest.mark.parametrize("N", [64, 300])
def test_matches_library_sdpa_without_rope(N):
    g = torch.Generator().manual_seed(N)
    q, k, v = (torch.randn(1, 2, N, 128, generator=g, dtype=torch.float64) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)
    ref_lse = torch.logsumexp((q @ k.transpose(-1, -2)) / math.sqrt(128), dim=-1)
    O, L = attention.joint_attention(q.numpy(), k.numpy(), v.numpy(), pos=None)
    assert np.max(np.abs(O - ref.reshape(-1, 128).numpy())) < 1e-12
    assert np.max(np.abs(L - ref_lse.reshape(-1).numpy())) < 1e-12


def test_rows_sum_to_one():
    # V = identity makes O the probability matrix itself
    rng = np.random.default_rng(5)
    N = D = 16
    q, k, _, pos = _rand_case(rng, N, D, (4, 6, 6))
    O, _ = attention.joint_attention(q[None, None] * 3, k[None, None] * 3, np.eye(N)[None, None], pos=pos,
                                     axes=(4, 6, 6))
    assert np.all(O >= 0)
    assert np.max(np.abs(O.sum(axis=1) - 1.0)) < 1e-15 * N


def test_zero_query_gives_column_mean_and_log_n():
    rng = np.random.default_rng(6)
    N, D = 200, 128
    q = np.zeros((N, D))
    k = rng.standard_normal((N, D))
    v = rng.standard_normal((N, D))
    pos = rng.integers(0, 50, size=(N, 3))
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos)
    assert np.max(np.abs(O - v.mean(axis=0)[None, :])) < 1e-13
    assert np.max(np.abs(L - math.log(N))) < 1e-13


def test_dominant_key_returns_its_value_row():
    rng = np.random.default_rng(7)
    N, D = 100, 128
    q = rng.standard_normal((N, D))
    k = rng.standard_normal((N, D)) * 0.05
    v = rng.standard_normal((N, D))
    i, j = 17, 63
    k[j] = 100.0 * math.sqrt(D) * q[i] / np.dot(q[i], q[i])     # logit 100 against |logit| < ~1
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None])
    assert np.max(np.abs(O[i] - v[j])) < 1e-12
    assert abs(L[i] - 100.0) < 1e-6


def test_joint_permutation_equivariance():
    rng = np.random.default_rng(8)
    N, D = 96, 128
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    pos = rng.integers(0, 40, size=(N, 3))
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos)
    perm = rng.permutation(N)
    # tokens keep their own position: permuting q, k, v and pos together permutes the rows of O
    O2, L2 = attention.joint_attention(q[perm][None, None], k[perm][None, None], v[perm][None, None], pos=pos[perm])
    assert np.max(np.abs(O2 - O[perm])) < 1e-12
    assert np.max(np.abs(L2 - L[perm])) < 1e-12
    # permuting keys and values jointly (queries fixed) changes nothing
    kp = k.copy()
    vp = v.copy()
    text = np.arange(32)
    pos_t = pos.copy()
    pos_t[text] = 0                       # text tokens all sit at position 0
    Ot, Lt = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos_t)
    sh = rng.permutation(32)
    kp[text] = k[sh]
    vp[text] = v[sh]
    Op, Lp = attention.joint_attention(q[None, None], kp[None, None], vp[None, None], pos=pos_t)
    assert np.max(np.abs(Op - Ot)) < 1e-12
    assert np.max(np.abs(Lp - Lt)) < 1e-12


def test_round_rotated_changes_only_operands():
    rng = np.random.default_rng(9)
    N, D = 64, 128
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    pos = rng.integers(0, 20, size=(N, 3))
    from oracle import formats
    phi = rope.angles(pos)
    qr = formats.round_bf16(rope.rotate(q, phi))
    kr = formats.round_bf16(rope.rotate(k, phi))
    O_ref, L_ref = attention.attention_rows(qr, kr, v, 1 / math.sqrt(D))
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos, round_rotated="bf16")
    assert np.array_equal(O, O_ref) and np.array_equal(L, L_ref)


# ---------------------------------------------------------------- rotary pins

def test_rope_preserves_pair_norms_and_is_identity_at_origin():
    rng = np.random.default_rng(10)
    N, D = 50, 128
    x = rng.standard_normal((N, D))
    pos = rng.integers(0, 128, size=(N, 3))
    pos[:5] = 0
    y = rope.rotate(x, rope.angles(pos))
    nx = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
    ny = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    assert np.max(np.abs(nx - ny)) < 1e-12
    assert np.array_equal(y[:5], x[:5])


def test_rope_relative_position():
    rng = np.random.default_rng(11)
    D = 128
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    for _ in range(10):
        m = rng.integers(0, 128, size=3)
        n = rng.integers(0, 128, size=3)
        lhs = np.dot(rope.rotate(q[None], rope.angles(m[None]))[0], rope.rotate(k[None], rope.angles(n[None]))[0])
        rhs = np.dot(q, rope.rotate(k[None], rope.angles((n - m)[None]))[0])
        assert abs(lhs - rhs) < 1e-11


@pytest.mark.parametrize("channel,axis,omega", [
    (0, 0, 1.0),                      # first t pair
    (14, 0, 10.0 ** -3.5),            # last t pair: 10000^(-14/16)
    (16, 1, 1.0),                     # first h pair
    (70, 1, 10.0 ** (-27.0 / 7.0)),   # last h pair: 10000^(-54/56)
    (72, 2, 1.0),                     # first w pair
    (126, 2, 10.0 ** (-27.0 / 7.0)),  # last w pair
    (40, 1, 10.0 ** (-96.0 / 56.0)),  # h pair 12: 10000^(-24/56)
])
def test_rope_single_pair_logit_is_cos_of_angle(channel, axis, omega):
    e = np.zeros(128)
    e[channel] = 1.0
    for delta in (1, 3, 17, 127):
        a = np.zeros(3, dtype=np.int64)
        b = np.zeros(3, dtype=np.int64)
        b[axis] = delta
        other = [x for x in range(3) if x != axis]
        a[other] = [5, 9]              # moving the other axes must not matter
        b[other] = [2, 100]
        qa = rope.rotate(e[None], rope.angles(a[None]))[0]
        kb = rope.rotate(e[None], rope.angles(b[None]))[0]
        assert abs(np.dot(qa, kb) - math.cos(delta * omega)) < 1e-13


def test_rope_rotation_direction():
    # (x, y) = (1, 0) turns to (cos phi, sin phi); (0, 1) turns to (-sin phi, cos phi)
    p = np.array([[0, 3, 0]])
    phi = 3.0                                  # first h pair, omega = 1
    ex = np.zeros(128)
    ex[16] = 1
    ey = np.zeros(128)
    ey[17] = 1
    rx = rope.rotate(ex[None], rope.angles(p))[0]
    ry = rope.rotate(ey[None], rope.angles(p))[0]
    assert abs(rx[16] - math.cos(phi)) < 1e-15 and abs(rx[17] - math.sin(phi)) < 1e-15
    assert abs(ry[16] + math.sin(phi)) < 1e-15 and abs(ry[17] - math.cos(phi)) < 1e-15


# --------------------------------------------------------------- merge pins

def test_merge_of_key_slices_equals_full_attention():
    rng = np.random.default_rng(12)
    N, D = 180, 128
    q, k, v = (rng.standard_normal((N, D)) * 2 for _ in range(3))
    full_o, full_l = attention.attention_rows(q, k, v, 1 / math.sqrt(D))
    cuts = [0, 50, 51, 130, N]
    parts = [attention.attention_rows(q, k[a:b], v[a:b], 1 / math.sqrt(D)) for a, b in zip(cuts[:-1], cuts[1:])]
    o, l = merge.merge([p[0] for p in parts], [p[1] for p in parts])
    assert np.max(np.abs(o - full_o)) < 1e-13
    assert np.max(np.abs(l - full_l)) < 1e-12
    o1, l1 = merge.merge([full_o], [full_l])
    assert np.max(np.abs(o1 - full_o)) < 1e-15 and np.max(np.abs(l1 - full_l)) < 1e-15


def test_merge_ignores_empty_key_slices():
    """A slice with no keys (sum exp = 0, lse = -inf, O = 0/0) changes
    nothing; the union of empty slices is empty (lse = -inf, O = 0)."""
    rng = np.random.default_rng(14)
    N, D = 40, 128
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    full_o, full_l = attention.attention_rows(q, k, v, 1 / math.sqrt(D))
    nan_o = np.full((N, D), np.nan)
    ninf = np.full(N, -np.inf)
    o, l = merge.merge([nan_o, full_o, nan_o], [ninf, full_l, ninf])
    assert np.array_equal(o, full_o) and np.array_equal(l, full_l)
    o, l = merge.merge([nan_o, nan_o], [ninf, ninf])
    assert np.array_equal(o, np.zeros((N, D))) and np.all(np.isneginf(l))
    # rows that are empty in one part only
    half = full_l.copy()
    half[::2] = -np.inf
    o, l = merge.merge([np.where(np.isneginf(half)[:, None], np.nan, full_o), full_o], [half, full_l])
    assert np.max(np.abs(o - full_o)) < 1e-15
    assert np.max(np.abs(l[1::2] - (full_l[1::2] + math.log(2)))) < 1e-13
    assert np.array_equal(l[::2], full_l[::2])


def test_merge_weights_follow_the_softmax_of_the_lses():
    """Two parts with scalar outputs 0 and 1: O is the logistic function of
    lse_1 - lse_0, and lse is log(e^a + e^b), both closed forms."""
    a = np.array([0.0, 3.0, -20.0, 700.0, -700.0])
    b = np.array([0.0, -1.0, 5.0, 700.5, -699.0])
    o, l = merge.merge([np.zeros((5, 1)), np.ones((5, 1))], [a, b])
    assert np.max(np.abs(o[:, 0] - 1.0 / (1.0 + np.exp(a - b)))) < 1e-15
    assert np.max(np.abs(l - np.logaddexp(a, b))) < 1e-12


# --------------------------------------------------------------- block-sparse pins

def _sparse_case(seed=21, B=1, H=2, N=700):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((B, H, N, 128)) for _ in range(3))
    pos = rng.integers(0, 40, size=(N, 3))
    nq, nk = -(-N // 512), -(-N // 128)
    return rng, q, k, v, pos, nq, nk


def test_all_ones_mask_is_dense_attention():
    rng, q, k, v, pos, nq, nk = _sparse_case()
    O, L = attention.joint_attention(q, k, v, pos=pos)
    Os, Ls = attention.joint_attention(q, k, v, pos=pos, kv_mask=np.ones((1, 2, nq, nk), np.uint8))
    assert np.array_equal(O, Os) and np.array_equal(L, Ls)


def test_single_tile_mask_is_attention_over_that_key_slice():
    rng, q, k, v, pos, nq, nk = _sparse_case()
    mask = np.zeros((1, 2, nq, nk), np.uint8)
    mask[0, 1, 0, 5] = 1                 # rows 0..511 of head 1 see keys 640..699 (the ragged last tile)
    mask[0, 1, 1, 2] = 1                 # rows 512..699 of head 1 see keys 256..383
    rows = np.array([[0, 1, 3], [0, 1, 511], [0, 1, 512], [0, 1, 699]])
    O, L = attention.joint_attention(q, k, v, pos=pos, rows=rows, kv_mask=mask)
    ang = rope.angles(pos)
    qr, kr = rope.rotate(q[0, 1], ang), rope.rotate(k[0, 1], ang)
    for i, (lo, hi) in enumerate([(640, 700), (640, 700), (256, 384), (256, 384)]):
        o, l = attention.attention_rows(qr[rows[i, 2]][None], kr[lo:hi], v[0, 1, lo:hi], 1 / math.sqrt(128))
        assert np.max(np.abs(O[i] - o[0])) < 1e-13 and abs(L[i] - l[0]) < 1e-12


def test_rows_without_keys_are_zero_with_minus_infinite_lse():
    rng, q, k, v, pos, nq, nk = _sparse_case()
    mask = np.ones((1, 2, nq, nk), np.uint8)
    mask[0, 0, 1, :] = 0
    O, L = attention.joint_attention(q, k, v, pos=pos, kv_mask=mask)
    O = O.reshape(1, 2, 700, 128)
    L = L.reshape(1, 2, 700)
    assert np.all(O[0, 0, 512:] == 0) and np.all(np.isneginf(L[0, 0, 512:]))
    assert np.all(np.isfinite(L[0, 0, :512])) and np.all(np.isfinite(L[0, 1]))


def test_complementary_masks_merge_to_dense_attention():
    """Splitting the key tiles of every row between two masks and merging the
    two block-sparse results gives the dense result: ties the block-sparse
    definition to the merge of partial results."""
    rng, q, k, v, pos, nq, nk = _sparse_case()
    m1 = rng.integers(0, 2, size=(1, 2, nq, nk)).astype(np.uint8)
    m1[0, 0, 0, :] = 0                   # one block entirely in the other part
    m2 = 1 - m1
    O, L = attention.joint_attention(q, k, v, pos=pos)
    O1, L1 = attention.joint_attention(q, k, v, pos=pos, kv_mask=m1)
    O2, L2 = attention.joint_attention(q, k, v, pos=pos, kv_mask=m2)
    Om, Lm = merge.merge([O1, O2], [L1, L2])
    assert np.max(np.abs(Om - O)) < 1e-13
    assert np.max(np.abs(Lm - L)) < 1e-12


def test_sampled_rows_equal_the_same_rows_of_the_full_result():
    rng = np.random.default_rng(13)
    B, H, N, D = 2, 3, 70, 128
    q, k, v = (rng.standard_normal((B, H, N, D)) for _ in range(3))
    pos = rng.integers(0, 30, size=(N, 3))
    O, L = attention.joint_attention(q, k, v, pos=pos)
    flat = rng.choice(B * H * N, 40, replace=False)          # unsorted, spread over (b, h)
    rows = np.stack([flat // (H * N), (flat // N) % H, flat % N], axis=1)
    Os, Ls = attention.joint_attention(q, k, v, pos=pos, rows=rows)
    assert np.max(np.abs(Os - O[flat])) < 1e-13
    assert np.max(np.abs(Ls - L[flat])) < 1e-13


def test_fp32_table_option_rounds_only_the_table():
    rng = np.random.default_rng(14)
    N, D = 40, 128
    q, k, v = (rng.standard_normal((N, D)) for _ in range(3))
    pos = rng.integers(0, 100, size=(N, 3))
    c, s = rope.table(pos)
    c32, s32 = rope.table_fp32(pos)
    # nearest fp32: within half an fp32 ulp of the fp64 value, and on the fp32 grid
    assert np.all(np.abs(c32 - c) <= 2.0 ** -25) and np.array_equal(c32, c32.astype(np.float32))
    from oracle import formats
    qr = formats.round_bf16(rope.rotate_with_table(q, c32, s32))
    kr = formats.round_bf16(rope.rotate_with_table(k, c32, s32))
    O_ref, L_ref = attention.attention_rows(qr, kr, v, 1 / math.sqrt(D))
    O, L = attention.joint_attention(q[None, None], k[None, None], v[None, None], pos=pos, round_rotated="bf16",
                                     table_fp32=True)
    assert np.array_equal(O, O_ref) and np.array_equal(L, L_ref)
