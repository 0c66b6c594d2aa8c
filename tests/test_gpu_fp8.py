"""Parity of the FP8 E4M3 path with the fp64 oracle.  Needs a B200.

* dit_attn_quantize_fp8 is bit-exact against the oracle's block quantiser
  applied to the oracle's fp32 rotation (q, k: fp32 table entries, products
  exact, evaluated in fp64 and rounded to fp32; v: no rotation).
* dit_attn_forward_fp8 is fed the ORACLE's codes and scales and compared with
  exact fp64 attention of the same dequantised values: relative L2 error of O
  <= 3e-2 (the FP8 variant's error budget), and, because P and the
  dequantised V stay in fp16 inside the kernel, also the BF16 path's
  max-abs 2e-2 / mean-abs 2e-3 and LSE bars.
* The end-to-end format floor (exact attention of the bf16 inputs against
  exact attention of their FP8 quantisation) is printed, not gated.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build
from oracle import attention as oracle_attention
from oracle import fp8 as oracle_fp8
from oracle import rope as oracle_rope

from gpu_cases import BF16_MAX_ABS, BF16_MEAN_ABS, errors, gather_rows, lse_bound, near_midpoint_blocks

pytestmark = pytest.mark.gpu

FP8_REL_L2 = 3e-2


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def oracle_fp32_operands(w, q, k, v, rope=True):
    """fp32 values the quantiser codes: rotated q, k (fp32 table), plain v."""
    q64, k64, v64 = (oracle_attention.to_f64(t) for t in (q, k, v))
    if rope:
        c, s = oracle_rope.table_fp32(W.positions(w))
        q64 = oracle_rope.rotate_with_table(q64, c, s)
        k64 = oracle_rope.rotate_with_table(k64, c, s)
    return q64.astype(np.float32), k64.astype(np.float32), v64.astype(np.float32)


def oracle_quantised(w, q, k, v, rope=True):
    """[(codes, scales)] for q, k, v, all from the oracle."""
    return [oracle_fp8.quantize(x) for x in oracle_fp32_operands(w, q, k, v, rope)]


def gpu_forward(quant, n_txt, out_f32=True, with_lse=True):
    dev = [(torch.from_numpy(c).cuda(), torch.from_numpy(s).cuda()) for c, s in quant]
    out, lse = dit.forward_fp8(dev[0][0], dev[1][0], dev[2][0], dev[0][1], dev[1][1], dev[2][1], n_txt=n_txt,
                               out_f32=out_f32, with_lse=with_lse)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    return out, lse


def oracle_on_codes(quant, rows):
    deq = [oracle_fp8.dequantize(c, s) for c, s in quant]
    return oracle_attention.joint_attention(deq[0], deq[1], deq[2], pos=None, rows=rows)


def rel_l2(got, ref):
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def check(out, lse, rows, O_ref, L_ref, label):
    got = gather_rows(out, rows)
    r = rel_l2(got, O_ref)
    mx, mean = errors(got, O_ref)
    dl = np.abs(gather_rows(lse, rows) - L_ref) if lse is not None else np.zeros(1)
    print("%s: rel-L2 %.3e max-abs %.3e mean-abs %.3e max|dLSE| %.3e (%d rows)" % (label, r, mx, mean, dl.max(),
                                                                                   len(rows)))
    assert r <= FP8_REL_L2, label
    assert mx <= BF16_MAX_ABS and mean <= BF16_MEAN_ABS, label
    if lse is not None:
        assert np.all(dl <= lse_bound(L_ref)), label


def check_quantiser(w, q, k, v, rope=True):
    ref = oracle_quantised(w, q, k, v, rope)
    cs = dit.rope_table(torch.from_numpy(W.positions(w)).cuda()) if rope else (None, None)
    for name, x, (codes, scales), rot in (("q", q, ref[0], True), ("k", k, ref[1], True), ("v", v, ref[2], False)):
        c8, sc = dit.quantize_fp8(x.cuda(), *(cs if rot else (None, None)))
        torch.cuda.synchronize()
        got_s = sc.cpu().numpy()
        got_c = c8.cpu().numpy()
        assert np.array_equal(got_s.view(np.uint32), scales.view(np.uint32)), "%s scales N=%d" % (name, w.N)
        bad = np.count_nonzero(got_c != codes)
        assert bad == 0, "%s: %d of %d codes differ (N=%d)" % (name, bad, codes.size, w.N)
    return ref


# ------------------------------------------------------------------ quantiser

@pytest.mark.parametrize("name", ["tiny_256", "t2i_512px"])
def test_quantiser_bitexact(name):
    w = W.WORKLOADS[name]
    check_quantiser(w, *W.make_qkv(w, seed=0))


QUANT_RAGGED = [(1, 1, 1, ()), (1, 2, 7, ((3, 5),)), (2, 1, 64, ((6, 6),)), (1, 3, 128, ((1, 1),))]


@pytest.mark.parametrize("B,H,n_txt,grids", QUANT_RAGGED)
def test_quantiser_ragged_bitexact(B, H, n_txt, grids):
    w = W.custom(B, H, n_txt, grids, outliers=True)
    check_quantiser(w, *W.make_qkv(w, seed=5))


def test_quantiser_zero_block_has_scale_one():
    w = W.custom(1, 1, 64, ((8, 8),))
    q, k, v = W.make_qkv(w, seed=6)
    v[..., :64, :] = 0          # first block all zero -> scale 1, codes 0
    codes, scales = dit.quantize_fp8(v.cuda())
    torch.cuda.synchronize()
    assert scales[0, 0, 0].item() == 1.0
    assert int(codes[..., :64, :].to(torch.int32).sum()) == 0
    check_quantiser(w, q, k, v)


def test_quantiser_bitexact_near_e4m3_midpoints():
    """Quotients x / scale on or within a few fp32 ulps of the midpoints
    between neighbouring E4M3 values, exact ties included (blocks with
    power-of-two scales): the codes are those of the correctly rounded fp32
    quotient, rounded to nearest even, and the scales amax / 448."""
    x = near_midpoint_blocks()
    codes_ref, scales_ref = oracle_fp8.quantize(x)
    assert oracle_fp8.tie_count(x, scales_ref) > 1000      # the ties are there
    xb = torch.from_numpy(x).to(torch.bfloat16)            # exact: every value is a bf16 value
    assert torch.equal(xb.float(), torch.from_numpy(x))
    codes, scales = dit.quantize_fp8(xb.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(scales.cpu().numpy(), scales_ref)
    assert np.array_equal(codes.cpu().numpy(), codes_ref)


# ------------------------------------------------------------------ attention

@pytest.fixture(scope="module")
def c4_case():
    w = W.WORKLOADS["t2i_2048px"]
    q, k, v = W.make_qkv(w, seed=0)
    return w, q, k, v


def test_quantiser_bitexact_outlier_2048(c4_case):
    w, q, k, v = c4_case
    check_quantiser(w, q, k, v)


@pytest.mark.parametrize("name", ["tiny_256", "t2i_512px", "t2i_2048px"])
def test_fp8_attention_parity(name, c4_case):
    if name == "t2i_2048px":
        w, q, k, v = c4_case
    else:
        w = W.WORKLOADS[name]
        q, k, v = W.make_qkv(w, seed=0)
    quant = oracle_quantised(w, q, k, v)
    rows = W.sample_rows(w)
    O_ref, L_ref = oracle_on_codes(quant, rows)
    out, lse = gpu_forward(quant, w.n_txt)
    check(out, lse, rows, O_ref, L_ref, name + " fp32-out vs oracle on the codes")
    out16, _ = gpu_forward(quant, w.n_txt, out_f32=False, with_lse=False)
    r16 = rel_l2(gather_rows(out16, rows), O_ref)
    assert r16 <= FP8_REL_L2
    # reported only: the format floor against exact attention of the bf16 inputs
    O_ex, _ = oracle_attention.joint_attention(q, k, v, pos=W.positions(w), rows=rows)
    print("%s: bf16-out rel-L2 %.3e; FP8 format floor vs exact bf16-input attention: oracle %.3e, kernel %.3e" % (
        name, r16, rel_l2(O_ref, O_ex), rel_l2(gather_rows(out, rows), O_ex)))


ATTN_RAGGED = [
    (1, 1, 1, ()),              # a single token
    (1, 1, 7, ((3, 5),)),       # N = 22 < one tile, one partial scale block
    (2, 3, 64, ((10, 10),)),    # N = 164: one full tile + 36
    (1, 2, 128, ((1, 1),)),     # N = 129: a tail tile of one key, a block of one token
    (2, 2, 77, ((13, 17), (5, 7))),   # N = 333
    (1, 1, 512, ((20, 20),)),   # N = 912
]


@pytest.mark.parametrize("B,H,n_txt,grids", ATTN_RAGGED)
def test_fp8_attention_ragged(B, H, n_txt, grids):
    w = W.custom(B, H, n_txt, grids, outliers=True)
    q, k, v = W.make_qkv(w, seed=7)
    quant = oracle_quantised(w, q, k, v)
    rows = W.sample_rows(w)
    O_ref, L_ref = oracle_on_codes(quant, rows)
    out, lse = gpu_forward(quant, w.n_txt)
    check(out, lse, rows, O_ref, L_ref, "ragged N=%d" % w.N)


def test_fp8_end_to_end_through_the_quantiser():
    """quantize_fp8 on the device feeding forward_fp8 equals forward_fp8 on
    the oracle's codes (the quantiser is bit-exact), bit for bit."""
    w = W.WORKLOADS["t2i_512px"]
    q, k, v = W.make_qkv(w, seed=0)
    cs = dit.rope_table(torch.from_numpy(W.positions(w)).cuda())
    q8, qs = dit.quantize_fp8(q.cuda(), *cs)
    k8, ks = dit.quantize_fp8(k.cuda(), *cs)
    v8, vs = dit.quantize_fp8(v.cuda())
    a, la = dit.forward_fp8(q8, k8, v8, qs, ks, vs, n_txt=w.n_txt, out_f32=True)
    b, lb = gpu_forward(oracle_quantised(w, q, k, v), w.n_txt)
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_fp8_reruns_bitwise_and_lse_optional():
    w = W.custom(1, 2, 40, ((12, 12),), outliers=True)
    quant = oracle_quantised(w, *W.make_qkv(w, seed=8))
    a, la = gpu_forward(quant, w.n_txt, out_f32=False)
    b, lb = gpu_forward(quant, w.n_txt, out_f32=False)
    c, _ = gpu_forward(quant, w.n_txt, out_f32=False, with_lse=False)
    assert torch.equal(a, b) and torch.equal(la, lb) and torch.equal(a, c)


def test_fp8_constant_values_give_constant_output():
    w = W.custom(1, 2, 40, ((9, 11),))
    q, k, v = W.make_qkv(w, seed=9)
    v[:] = torch.linspace(-3, 3, 128, dtype=torch.float32).to(torch.bfloat16)
    quant = oracle_quantised(w, q, k, v)
    out, _ = gpu_forward(quant, w.n_txt)
    vdq = torch.from_numpy(oracle_fp8.dequantize(*quant[2])[0, 0, 0]).float()
    # every V row dequantises to the same values; softmax weights sum to one
    assert torch.allclose(out.cpu(), vdq.expand_as(out.cpu()), atol=2e-3, rtol=1e-3)


@pytest.mark.parametrize("p", [0, 63, 64, 65, 67, 127, 128, 199])
def test_fp8_dominant_key_across_scale_blocks(p):
    """One key whose logit dominates by ~200 while the key blocks' scales
    differ by 1e4: the row returns that key's value row, so each half tile's
    maximum is taken with its own block's scale."""
    B, H, N = 1, 1, 200
    nb = (N + 63) // 64
    q8 = np.full((B, H, N, 128), 0x7E, dtype=np.uint8)            # 448
    k8 = np.zeros((B, H, N, 128), dtype=np.uint8)
    k8[0, 0, p] = 0x7E
    ks = np.ones((B, H, nb), dtype=np.float32)
    ks[0, 0, p // 64] = 1e-4                   # logit of key p: 128 * 448^2 * 1e-4 / sqrt(128) ~ 227
    rng = np.random.default_rng(p)
    v8 = rng.integers(0, 0x7F, size=(B, H, N, 128), dtype=np.uint8)   # codes below the NaN pattern
    ones = np.ones((B, H, nb), dtype=np.float32)
    quant = [(q8, ones), (k8, ks), (v8, ones)]
    out, lse = gpu_forward(quant, 0)
    from oracle import formats
    want = formats.e4m3_decode(v8[0, 0, p])
    got = out[0, 0].double().cpu().numpy()
    assert np.isfinite(got).all()
    assert np.array_equal(got, np.broadcast_to(want, got.shape))
