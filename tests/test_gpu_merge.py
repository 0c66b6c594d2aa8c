"""Parity of dit_attn_merge (partial results over disjoint key sets) with the
oracle's merge.  Needs a B200.

Inputs are partial results of exact attention over key slices, computed by
the oracle, so the merged result is also the attention over all keys.  Bars:
fp32 output within d = 1e-5 (1 + |O|) of the oracle, lse within 1e-5 (1 + |lse|)
(fp32 weights from expf / logf); a bf16 output is additionally rounded once,
so it gets 2^-8 (|O| + d) on top.  Single parts, empty parts and in-place merges
have exact expected values.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build
from oracle import attention as oracle_attention
from oracle import formats
from oracle import merge as oracle_merge

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def key_slice_parts(w, cuts, seed=0):
    """Oracle partial (O_r, lse_r) of every row of w over the key slices cuts."""
    q, k, v = W.make_qkv(w, seed)
    pos = W.positions(w)
    from oracle import rope
    q64 = rope.rotate(oracle_attention.to_f64(q), rope.angles(pos))
    k64 = rope.rotate(oracle_attention.to_f64(k), rope.angles(pos))
    v64 = oracle_attention.to_f64(v)
    scale = 1 / np.sqrt(w.D)
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        O = np.empty((w.B, w.H, w.N, w.D))
        L = np.empty((w.B, w.H, w.N))
        for bi in range(w.B):
            for h in range(w.H):
                O[bi, h], L[bi, h] = oracle_attention.attention_rows(q64[bi, h], k64[bi, h, a:b], v64[bi, h, a:b],
                                                                     scale)
        parts.append((O, L))
    return parts


def to_dev(parts, part_f32):
    dt = torch.float32 if part_f32 else torch.bfloat16
    return ([torch.from_numpy(o).to(dt).cuda() for o, _ in parts],
            [torch.from_numpy(l).float().cuda() for _, l in parts])


def oracle_on(o_dev, l_dev):
    """Oracle merge of the parts' own values, row by row ([..., D] parts)."""
    shape = tuple(o_dev[0].shape)
    outs = [o.double().cpu().numpy().reshape(-1, shape[-1]) for o in o_dev]
    lses = [l.double().cpu().numpy().reshape(-1) for l in l_dev]
    O, L = oracle_merge.merge(outs, lses)
    return O.reshape(shape), L.reshape(shape[:-1])


def check(out, lse, O_ref, L_ref, out_f32, label):
    got = out.double().cpu().numpy()
    # fp32 result within d of the oracle; a bf16 store then moves y by at most
    # half a bf16 spacing, <= 2^-8 |y| with |y| <= |O_ref| + d
    d = 1e-5 * (1 + np.abs(O_ref))
    tol = d + (0 if out_f32 else 2.0 ** -8 * (np.abs(O_ref) + d))
    err = np.abs(got - O_ref)
    print("%s: max |dO| %.3e (max |dO| / tol %.3f)" % (label, err.max(), (err / tol).max()))
    assert np.all(err <= tol), label
    if lse is not None:
        gl = lse.double().cpu().numpy()
        fin = np.isfinite(L_ref)
        assert np.array_equal(np.isneginf(gl), np.isneginf(L_ref))
        assert np.all(np.abs(gl[fin] - L_ref[fin]) <= 1e-5 * (1 + np.abs(L_ref[fin]))), label


@pytest.mark.parametrize("part_f32", [True, False])
@pytest.mark.parametrize("out_f32", [True, False])
def test_merge_of_key_slices(part_f32, out_f32):
    w = W.WORKLOADS["tiny_256"]
    cuts = [0, 64, 100, 101, 256]
    parts = key_slice_parts(w, cuts)
    o_dev, l_dev = to_dev(parts, part_f32)
    out, lse = dit.merge(o_dev, l_dev, out_f32=out_f32)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_on(o_dev, l_dev)
    check(out, lse, O_ref, L_ref, out_f32, "R=%d part_f32=%s out_f32=%s" % (len(parts), part_f32, out_f32))
    # and the merge of the key slices is the attention over all keys
    O_full, L_full = key_slice_parts(w, [0, w.N])[0]
    if part_f32 and out_f32:
        assert np.max(np.abs(out.double().cpu().numpy() - O_full)) < 1e-5 * (1 + np.abs(O_full).max())
        assert np.max(np.abs(lse.double().cpu().numpy() - L_full)) < 1e-4


@pytest.mark.parametrize("R", [1, 2, 3, 16])
def test_merge_part_counts_and_ragged_rows(R):
    """Random parts on a ragged row count (rows not a multiple of the 16 rows
    of a CTA), lse spread over +-40 so the weights span many decades."""
    rng = np.random.default_rng(R)
    B, H, N = 2, 3, 37
    o = [torch.from_numpy(rng.standard_normal((B, H, N, 128)) * 3).float().cuda() for _ in range(R)]
    l = [torch.from_numpy(rng.uniform(-40, 40, (B, H, N))).float().cuda() for _ in range(R)]
    out, lse = dit.merge(o, l, out_f32=True)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_on(o, l)
    check(out, lse, O_ref, L_ref, True, "R=%d random" % R)


def test_single_part_is_returned_exactly():
    rng = np.random.default_rng(3)
    o = torch.from_numpy(rng.standard_normal((1, 2, 50, 128))).float().cuda()
    l = torch.from_numpy(rng.standard_normal((1, 2, 50)) * 10).float().cuda()
    out, lse = dit.merge([o], [l], out_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(out, o) and torch.equal(lse, l)
    ob = o.to(torch.bfloat16)
    out_b, _ = dit.merge([ob], [l])
    torch.cuda.synchronize()
    assert torch.equal(out_b, ob)


def test_empty_parts_are_ignored():
    rng = np.random.default_rng(4)
    B, H, N = 1, 2, 40
    o0 = torch.from_numpy(rng.standard_normal((B, H, N, 128))).float().cuda()
    l0 = torch.from_numpy(rng.standard_normal((B, H, N))).float().cuda()
    nan_o = torch.full_like(o0, float("nan"))
    ninf = torch.full_like(l0, float("-inf"))
    out, lse = dit.merge([nan_o, o0, nan_o], [ninf, l0, ninf], out_f32=True)
    torch.cuda.synchronize()
    assert torch.equal(out, o0) and torch.equal(lse, l0)
    # rows empty in every part
    l1 = l0.clone()
    l1[0, 1, ::3] = float("-inf")
    o1 = torch.where(torch.isneginf(l1)[..., None], nan_o, o0)
    out, lse = dit.merge([o1, nan_o], [l1, ninf], out_f32=True)
    torch.cuda.synchronize()
    O_ref, L_ref = oracle_on([o1, nan_o], [l1, ninf])
    assert np.array_equal(out.double().cpu().numpy(), O_ref)
    assert np.array_equal(np.isneginf(lse.cpu().numpy()), np.isneginf(L_ref))


def test_in_place_merge():
    rng = np.random.default_rng(5)
    o = [torch.from_numpy(rng.standard_normal((1, 2, 77, 128))).float().cuda() for _ in range(3)]
    l = [torch.from_numpy(rng.standard_normal((1, 2, 77)) * 5).float().cuda() for _ in range(3)]
    want, want_l = dit.merge(o, l, out_f32=True)
    dit.dit_attn_merge(o, l, o[1], l[2], dit.DIT_PART_F32 | dit.DIT_OUT_F32)
    torch.cuda.synchronize()
    assert torch.equal(o[1], want) and torch.equal(l[2], want_l)


def test_merge_at_2048px_size_on_sampled_rows():
    """Two bf16 parts of the 2048x2048 shape (B=1, H=24, N=16896), as a 2-way
    context-parallel split would give; checked on the sampled rows."""
    w = W.WORKLOADS["t2i_2048px"]
    g = torch.Generator(device="cpu").manual_seed(6)
    shape = (w.B, w.H, w.N, 128)
    o = [(torch.randn(shape, generator=g) * 2).to(torch.bfloat16).cuda() for _ in range(2)]
    l = [(torch.randn(shape[:3], generator=g) * 8).cuda() for _ in range(2)]
    out, lse = dit.merge(o, l)
    torch.cuda.synchronize()
    rows = W.sample_rows(w)
    idx = torch.from_numpy(rows).cuda()
    pick = lambda t: t[idx[:, 0], idx[:, 1], idx[:, 2]]
    O_ref, L_ref = oracle_merge.merge([pick(x).double().cpu().numpy() for x in o],
                                      [pick(x).double().cpu().numpy() for x in l])
    check(pick(out), pick(lse), O_ref, L_ref, False, "2048px R=2 bf16")
