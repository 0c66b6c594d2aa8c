"""The QKV projection with the FP8 operand epilogue (dit_qkv_project_fp8)
against the fp64 oracle.  Needs a B200.

The kernel sums the C products of every output in fp32 in the tensor cores'
order, which no plain definition reproduces, so the gates are bounds derived
from that arithmetic rather than bit equality:

* |y_gpu - y| <= e = 2^-23 * C * M + 2^-23 |y|, with M = sum_c |x_c w_c| (the
  oracle's magnitude(): any order of C fp32 additions of exact products is
  within (C - 1) 2^-24 M when rounded, twice that when chopped, and the
  fp32 accumulator and the bias addition round once more each); the
  rotation of a pair adds at most the errors of both components plus one fp32
  rounding;
* the block scale is within the largest bound of its block / 448 (+1 ulp) of
  amax / 448 of the exact rotated values;
* every code, dequantised, is within half an E4M3 step (relative 2^-4, or
  2^-10 absolute in the subnormal range) times the GPU scale, plus the bound,
  of the exact rotated value: the code is the nearest one to y_gpu / scale;
* nearly every code equals the nearest code of the exact value (reported,
  and gated at 99.9 %);
* the optional bf16 outputs are within half a bf16 step plus the bound.
Then the codes feed dit_attn_forward_fp8, checked like the FP8 tests.
"""
import numpy as np
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build
from oracle import attention as oracle_attention, formats, fp8 as oracle_fp8, projection, rope as oracle_rope

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def _inputs(B, N, C, H, seed, bias=True):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, N, C, generator=g).to(torch.bfloat16)
    w = (torch.randn(3 * H * 128, C, generator=g) / np.sqrt(C)).to(torch.bfloat16)
    b = (0.1 * torch.randn(3 * H * 128, generator=g)).float() if bias else None
    return x, w, b


def _e4m3_half_step(v):
    """Half the E4M3 spacing at |v| (v in code units): 2^(e-4) for normal
    values, 2^-10 in the subnormal range."""
    a = np.abs(v)
    _, e = np.frexp(np.maximum(a, 2.0 ** -6))
    return np.ldexp(1.0, e - 1 - 4)


def _check_projection(B, N, C, H, seed, rope=True, bias=True, with_bf16=True, attend=False):
    x, w, bias_t = _inputs(B, N, C, H, seed, bias)
    pos = None
    if rope:
        # a joint sequence: text tokens, then an image grid 16 tokens wide
        rows = (N - N // 5) // 16
        pos = W.positions(W.custom(1, 1, N - 16 * rows, ((rows, 16),)))
        assert pos.shape[0] == N
    dev = torch.device("cuda")
    cs = dit.rope_table(torch.from_numpy(pos).to(dev)) if rope else (None, None)
    out = dit.qkv_project_fp8(x.to(dev), w.to(dev), None if bias_t is None else bias_t.to(dev), cs[0], cs[1],
                              with_bf16=with_bf16)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    codes = [t.cpu().numpy() for t in out[:3]]
    scales = [t.cpu().numpy().astype(np.float64) for t in out[3:6]]
    ys = projection.project(x, w, bias_t, H=H)
    mags = projection.magnitude(x, w, H=H)
    worst_match = 1.0
    for s in range(3):
        y, m = ys[s], mags[s]
        err = 2.0 ** -23 * C * m + 2.0 ** -23 * np.abs(y)
        if rope and s < 2:
            c, sn = oracle_rope.table_fp32(pos)
            r = oracle_rope.rotate_with_table(y, c, sn)
            e_pair = err[..., 0::2] + err[..., 1::2]
            err = np.repeat(e_pair, 2, axis=-1) + 2.0 ** -24 * np.abs(r)
        else:
            r = y
        # block scales
        nb = (N + 63) // 64
        pad = nb * 64 - N
        rp = np.pad(np.abs(r), ((0, 0), (0, 0), (0, pad), (0, 0)))
        ep = np.pad(err, ((0, 0), (0, 0), (0, pad), (0, 0)))
        amax = rp.reshape(B, H, nb, -1).max(axis=-1)
        emax = ep.reshape(B, H, nb, -1).max(axis=-1)
        ref_scale = np.where(amax == 0, 1.0, amax / 448.0)
        assert np.all(np.abs(scales[s] - ref_scale) <= emax / 448.0 + 2.0 ** -22 * ref_scale), s
        # codes: dequantised within half a step (of the GPU scale) plus the bound
        sc = np.repeat(scales[s], 64, axis=2)[:, :, :N, None]
        deq = formats.e4m3_decode(codes[s]) * sc
        half = _e4m3_half_step(deq / sc) * sc
        assert np.all(np.abs(deq - r) <= half + err + 1e-30), s
        # agreement with the nearest code of the exact value
        match = float(np.mean(formats.e4m3_encode(r / sc) == codes[s]))
        worst_match = min(worst_match, match)
        if with_bf16:
            y16 = out[6 + s].double().cpu().numpy()
            assert np.all(np.abs(y16 - y) <= np.ldexp(1.0, np.frexp(np.abs(y))[1] - 9) + err), s
    print("projection B=%d N=%d C=%d H=%d: codes equal to the exact value's nearest code: %.5f" % (
        B, N, C, H, worst_match))
    assert worst_match >= 0.999
    if attend:
        q8, k8, v8, qs, ks, vs = out[:6]
        o, _ = dit.forward_fp8(q8, k8, v8, qs, ks, vs, out_f32=True)
        torch.cuda.synchronize()
        deq = [oracle_fp8.dequantize(a.cpu().numpy(), b.cpu().numpy()) for a, b in ((q8, qs), (k8, ks), (v8, vs))]
        rows = W.sample_rows(W.custom(B, H, N, ()))
        ref, _ = oracle_attention.joint_attention(deq[0], deq[1], deq[2], rows=rows)
        got = o.double().cpu().numpy()
        g = got[rows[:, 0], rows[:, 1], rows[:, 2]]
        rel = np.linalg.norm(g - ref) / np.linalg.norm(ref)
        print("FP8 attention on the projected codes: rel-L2 %.3e" % rel)
        assert rel <= 3e-2


def test_projection_small_ragged():
    # one-CTA tiles (H = 2); N not a multiple of the 128-token tile or of the 64-token block; C not a
    # multiple of 64
    _check_projection(B=2, N=300, C=200, H=2, seed=1)


def test_projection_pair_tiles_small_ragged():
    # H a multiple of 4: CTA pairs of 256 tokens x 512 features; the second CTA of the last pair
    # holds tokens past N
    _check_projection(B=2, N=300, C=200, H=4, seed=4)


def test_projection_without_rope_or_bias():
    _check_projection(B=1, N=128, C=64, H=2, seed=2, rope=False, bias=False, with_bf16=False)


def test_projection_flux_hidden_size_feeds_the_fp8_attention():
    # FLUX width: C = 3072 = 24 heads x 128; the 512^2 joint sequence (512 text + 32x32 image tokens)
    _check_projection(B=1, N=1536, C=3072, H=24, seed=3, attend=True)
