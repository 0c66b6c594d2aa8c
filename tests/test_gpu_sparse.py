"""Parity of dit_attn_forward_sparse (block-sparse key tiles) with the fp64
oracle's block-sparse attention.  Needs a B200.

Bars as for the dense BF16 path: the fp32 output against the oracle whose
rotated q, k are rounded to bf16 (fp32 table entries), max-abs 2e-2,
mean-abs 2e-3, |dLSE| <= 1e-3 + 1e-5 |LSE|; rows whose query block selects no
key tile must be exactly 0 with LSE = -inf.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build
from oracle import attention as oracle_attention

from gpu_cases import BF16_MAX_ABS, BF16_MEAN_ABS, device_inputs, errors, gather_rows, lse_bound, rope_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def mask_shape(w):
    return (w.B, w.H, (w.N + 511) // 512, (w.N + 127) // 128)


def random_mask(w, density, seed):
    rng = np.random.default_rng(seed)
    return (rng.random(mask_shape(w)) < density).astype(np.uint8)


def prepared(w, inputs):
    q, k, v, qd, kd, vd = inputs
    c, s = rope_tables(w)
    kr = torch.empty_like(kd)
    v16 = torch.empty(vd.shape, dtype=torch.float16, device=vd.device)
    dit.dit_attn_prepare_kv(kd, vd, c, s, kr, v16)
    return qd, kr, v16, c, s


def run_sparse(w, inputs, mask, out_f32=True, fused=False):
    md = torch.from_numpy(mask).cuda()
    if fused:
        q, k, v, qd, kd, vd = inputs
        c, s = rope_tables(w)
        out, lse = dit.forward_sparse(qd, kd, vd, md, c, s, n_txt=w.n_txt, out_f32=out_f32)
    else:
        qd, kr, v16, c, s = prepared(w, inputs)
        out, lse = dit.forward_sparse(qd, kr, v16, md, c, s, n_txt=w.n_txt, out_f32=out_f32, k_rotated=True,
                                      v_f16=True)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    return out, lse


def check(w, inputs, mask, out, lse, rows, label):
    q, k, v = inputs[:3]
    O_ref, L_ref = oracle_attention.joint_attention(q, k, v, pos=W.positions(w), rows=rows, round_rotated="bf16",
                                                    table_fp32=True, kv_mask=mask)
    got, gl = gather_rows(out, rows), gather_rows(lse, rows)
    empty = np.isneginf(L_ref)
    assert np.array_equal(np.isneginf(gl), empty), label
    assert np.all(got[empty] == 0), label
    live = ~empty
    if live.any():
        mx, mean = errors(got[live], O_ref[live])
        dl = np.abs(gl[live] - L_ref[live])
        print("%s: %d rows (%d without keys): max-abs %.3e mean-abs %.3e max|dLSE| %.3e" % (
            label, len(rows), int(empty.sum()), mx, mean, dl.max()))
        assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, label
        assert np.all(dl <= lse_bound(L_ref[live])), label


def test_all_ones_mask_equals_dense_forward_bitwise():
    for name, fused in (("t2i_512px", False), ("tiny_256", True)):
        w = W.WORKLOADS[name]
        inputs = device_inputs(w)
        ones = np.ones(mask_shape(w), np.uint8)
        a, la = run_sparse(w, inputs, ones, fused=fused)
        if fused:
            b, lb = dit.forward(inputs[3], inputs[4], inputs[5], *rope_tables(w), n_txt=w.n_txt, out_f32=True)
        else:
            qd, kr, v16, c, s = prepared(w, inputs)
            b, lb = dit.forward(qd, kr, v16, c, s, n_txt=w.n_txt, out_f32=True, k_rotated=True, v_f16=True)
        torch.cuda.synchronize()
        assert torch.equal(a, b) and torch.equal(la, lb), name


SPARSE_CASES = [
    ("t2i_512px", 0.5, 11),
    ("t2i_1024px_cfg", 0.3, 12),
    ("t2i_1024px_cfg", 0.8, 13),
]


@pytest.mark.parametrize("name,density,seed", SPARSE_CASES)
def test_random_masks_match_oracle(name, density, seed):
    w = W.WORKLOADS[name]
    inputs = device_inputs(w, seed=seed)
    mask = random_mask(w, density, seed)
    mask[0, 0, 0, :] = 0                 # one query block with no key tile
    out, lse = run_sparse(w, inputs, mask)
    rows = W.sample_rows(w)
    rows = np.concatenate([rows, [[0, 0, 0], [0, 0, 17], [0, 0, 511]]])
    check(w, inputs, mask, out, lse, rows, "%s density %.1f" % (name, density))


RAGGED = [
    (1, 2, 7, ((3, 5),)),               # N = 22: one partial tile
    (2, 2, 77, ((13, 17), (5, 7))),     # N = 333: last tile of 77 keys
    (1, 1, 512, ((20, 20),)),           # N = 912: two query blocks, last of 400 rows
]


@pytest.mark.parametrize("B,H,n_txt,grids", RAGGED)
def test_ragged_shapes_both_modes(B, H, n_txt, grids):
    w = W.custom(B, H, n_txt, grids, outliers=True)
    inputs = device_inputs(w, seed=14)
    mask = random_mask(w, 0.6, 14)
    mask[..., -1] = 1                    # the ragged last tile selected everywhere ...
    mask[0, 0, 0, -1] = 0                # ... except for one block
    rows = W.sample_rows(w)
    for fused in (False, True):
        out, lse = run_sparse(w, inputs, mask, fused=fused)
        check(w, inputs, mask, out, lse, rows, "N=%d %s" % (w.N, "fused" if fused else "prepared"))


def test_empty_mask_gives_zero_output_and_minus_infinite_lse():
    w = W.custom(1, 2, 64, ((10, 10),))
    inputs = device_inputs(w, seed=15)
    out, lse = run_sparse(w, inputs, np.zeros(mask_shape(w), np.uint8), out_f32=False)
    assert torch.count_nonzero(out).item() == 0
    assert torch.isneginf(lse).all().item()


def test_complementary_masks_merge_to_dense():
    """Two block-sparse launches over complementary tile sets, merged on the
    GPU with dit_attn_merge, give the dense forward's result."""
    w = W.WORKLOADS["t2i_1024px_cfg"]
    inputs = device_inputs(w, seed=16)
    m1 = random_mask(w, 0.5, 16)
    m1[0, 1, 2, :] = 0
    m2 = (1 - m1).astype(np.uint8)
    o1, l1 = run_sparse(w, inputs, m1)
    o2, l2 = run_sparse(w, inputs, m2)
    merged, lm = dit.merge([o1, o2], [l1, l2], out_f32=True)
    qd, kr, v16, c, s = prepared(w, inputs)
    dense, ld = dit.forward(qd, kr, v16, c, s, n_txt=w.n_txt, out_f32=True, k_rotated=True, v_f16=True)
    torch.cuda.synchronize()
    err = ((merged - dense).abs() / (dense.abs() + 1)).max().item()
    print("merged halves vs dense: max |dO| / (|O| + 1) = %.2e, max |dLSE| = %.2e" % (
        err, (lm - ld).abs().max().item()))
    assert err <= 2e-3                   # P is rounded to fp16 relative to different running maxima
    assert (lm - ld).abs().max().item() <= 1e-3 + 1e-5 * ld.abs().max().item()


def test_sparse_2048px_sampled_rows():
    w = W.WORKLOADS["t2i_2048px"]
    inputs = device_inputs(w, seed=17)
    mask = random_mask(w, 0.5, 17)
    out, lse = run_sparse(w, inputs, mask)
    rows = W.sample_rows(w, count=2048)
    check(w, inputs, mask, out, lse, rows, "2048px density 0.5")
