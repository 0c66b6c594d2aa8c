"""Parity of the split form (compensated q~ k~^T on fp16 hi + lo operands,
DIT_QK_SPLIT) with the EXACT fp64 oracle on every workload, including the
two with x16 outlier channels, and the bound that keeps the default bf16-
operand path within its operand-rounding floor there.  Needs a B200.

Bars (the library's BF16 parity bars): max-abs <= 2e-2 and mean-abs <= 2e-3
on every checked output element, |dLSE| <= 1e-3 + 1e-5 |LSE|, all against
the oracle that rotates and attends in fp64 on the bf16 inputs.  The outlier
workloads are gated on the fp32-output path: their |O| reaches ~55, where
the bf16 spacing (0.25) alone exceeds 2e-2 whatever the kernel does.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build
from oracle import formats, rope as oracle_rope

from gpu_cases import (BF16_MAX_ABS, BF16_MEAN_ABS, device_inputs, errors, gather_rows, lse_bound, oracle_rows,
                       rope_tables, run_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def run_split(w, inputs, rope=True, out_f32=True):
    _, _, _, qd, kd, vd = inputs
    c, s = rope_tables(w) if rope else (None, None)
    k_split, v16 = dit.prepare_kv_split(kd, vd, c, s)
    out, lse = dit.forward(qd, k_split, v16, c, s, n_txt=w.n_txt, out_f32=out_f32, qk_split=True)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    return out, lse


def check(out, lse, rows, O_ref, L_ref, label):
    got = gather_rows(out, rows)
    mx, mean = errors(got, O_ref)
    dl = np.abs(gather_rows(lse, rows) - L_ref)
    ratio = float((dl / lse_bound(L_ref)).max())
    print("%s: max-abs %.3e mean-abs %.3e max|dLSE|/bound %.3f (%d rows)" % (label, mx, mean, ratio, len(rows)))
    assert mx <= BF16_MAX_ABS, label
    assert mean <= BF16_MEAN_ABS, label
    assert ratio <= 1.0, label


@pytest.mark.parametrize("name", ["tiny_256", "t2i_2048px"])
def test_prepare_kv_split_is_bit_exact(name):
    """hi / lo planes equal the oracle's split of RN32(RN64(rotation)) element
    for element (all heads), and v_f16 is v's fp16 cast."""
    w = W.WORKLOADS[name]
    _, k, v, _, kd, vd = device_inputs(w)
    c, s = rope_tables(w)
    k_split, v16 = dit.prepare_kv_split(kd, vd, c, s)
    torch.cuda.synchronize()
    tc, ts = oracle_rope.table_fp32(W.positions(w))
    for b in range(w.B):
        for h in range(w.H):
            hi, lo = oracle_rope.rotate_split(k[b, h].double().numpy(), tc, ts)
            assert np.array_equal(k_split[0, b, h].double().cpu().numpy(), hi), (b, h)
            assert np.array_equal(k_split[1, b, h].double().cpu().numpy(), lo), (b, h)
    assert torch.equal(v16, vd.to(torch.float16))
    # without tables: the split of k itself (bf16 values are exact in fp16 here: lo = 0)
    k_plain, _ = dit.prepare_kv_split(kd, vd)
    torch.cuda.synchronize()
    hi, lo = formats.split_fp16(k[0, 0].double().numpy())
    assert np.array_equal(k_plain[0, 0, 0].double().cpu().numpy(), hi)
    assert np.array_equal(k_plain[1, 0, 0].double().cpu().numpy(), lo)


@pytest.mark.parametrize("name", ["tiny_256", "t2i_512px", "t2i_1024px_cfg", "t2i_2048px", "i2i_2048px"])
def test_split_form_meets_the_bars_against_the_exact_oracle(name):
    w = W.WORKLOADS[name]
    inputs = device_inputs(w)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    O_ex, L_ex = oracle_rows(w, q, k, v, rows)
    out32, lse32 = run_split(w, inputs)
    check(out32, lse32, rows, O_ex, L_ex, name + " split fp32-out vs exact")
    out16, lse16 = run_split(w, inputs, out_f32=False)
    if not w.outliers:
        check(out16, lse16, rows, O_ex, L_ex, name + " split bf16-out vs exact")
    else:
        print("%s split bf16-out vs exact (bf16 format floor, reported): max/mean %.3e/%.3e" % (
            (name,) + errors(gather_rows(out16, rows), O_ex)))


RAGGED = [
    (1, 1, 1, ()),
    (1, 1, 7, ((3, 5),)),
    (2, 3, 64, ((10, 10),)),
    (1, 2, 128, ((1, 1),)),
    (2, 2, 77, ((13, 17), (5, 7))),
    (1, 1, 512, ((20, 20),)),
]


@pytest.mark.parametrize("B,H,n_txt,grids", RAGGED)
def test_split_form_ragged_shapes(B, H, n_txt, grids):
    w = W.custom(B, H, n_txt, grids, outliers=True)
    inputs = device_inputs(w, seed=5)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    O_ex, L_ex = oracle_rows(w, q, k, v, rows)
    out, lse = run_split(w, inputs)
    check(out, lse, rows, O_ex, L_ex, "split ragged N=%d" % w.N)


def test_split_form_without_rope_and_reruns_bitwise():
    w = W.custom(1, 3, 100, ((20, 20),), outliers=True)
    inputs = device_inputs(w, seed=6)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    O_ex, L_ex = oracle_rows(w, q, k, v, rows, rope=False)
    a, la = run_split(w, inputs, rope=False)
    check(a, la, rows, O_ex, L_ex, "split no rope")
    b, lb = run_split(w, inputs, rope=False)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("name", ["t2i_2048px", "i2i_2048px"])
def test_default_path_stays_within_its_operand_rounding_floor(name):
    """The bf16-operand path cannot meet the bars against the exact oracle on
    the outlier workloads (its operand rounding alone moves O by several
    units); gate its exact-oracle error at 1.1x that floor (max and mean),
    with the floor measured by the oracle itself: exact attention on the
    bf16-rounded rotated operands against exact attention."""
    w = W.WORKLOADS[name]
    inputs = device_inputs(w)
    q, k, v = inputs[:3]
    rows = W.sample_rows(w)
    O_ex, _ = oracle_rows(w, q, k, v, rows)
    O_op, _ = oracle_rows(w, q, k, v, rows, operands="bf16")
    floor_max, floor_mean = errors(O_op, O_ex)
    out32, _ = run_gpu(w, out_f32=True, inputs=inputs)
    mx, mean = errors(gather_rows(out32, rows), O_ex)
    print("%s default path vs exact: max %.3e mean %.3e; operand floor max %.3e mean %.3e" % (
        name, mx, mean, floor_max, floor_mean))
    assert mx <= 1.1 * floor_max and mean <= 1.1 * floor_mean
