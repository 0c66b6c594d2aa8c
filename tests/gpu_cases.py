"""Shared helpers of the GPU parity tests: run the CUDA path on a workload and
evaluate the fp64 oracle on the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from oracle import attention as oracle_attention
from oracle import formats

# Parity bars of the BF16 path (max-abs / mean-abs over all checked output
# elements; LSE in natural-log units of the scaled logits).
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3


def lse_bound(lse_ref):
    return 1e-3 + 1e-5 * np.abs(lse_ref)


def device_inputs(w, seed=0):
    q, k, v = W.make_qkv(w, seed)
    return q, k, v, q.cuda(), k.cuda(), v.cuda()


def rope_tables(w):
    pos = torch.from_numpy(W.positions(w)).cuda()
    return dit.rope_table(pos)


def gather_rows(t, rows):
    """t: [B, H, N, ...] tensor; rows: int [R, 3] (b, h, n) -> numpy [R, ...] fp64."""
    idx = torch.from_numpy(rows).to(t.device)
    return t[idx[:, 0], idx[:, 1], idx[:, 2]].double().cpu().numpy()


def errors(got, ref):
    e = np.abs(got - ref)
    return float(e.max()), float(e.mean())


def run_gpu(w, rope=True, out_f32=False, seed=0, inputs=None, prepared=True):
    """prepared: K / V go through dit_attn_prepare_kv first (the fast path);
    otherwise the kernel rotates K and converts V tile by tile."""
    if inputs is None:
        inputs = device_inputs(w, seed)
    q, k, v, qd, kd, vd = inputs
    cs = rope_tables(w) if rope else (None, None)
    if prepared and rope:
        kr = torch.empty_like(kd)
        v16 = torch.empty(vd.shape, dtype=torch.float16, device=vd.device)
        dit.dit_attn_prepare_kv(kd, vd, cs[0], cs[1], kr, v16)
        out, lse = dit.forward(qd, kr, v16, cs[0], cs[1], n_txt=w.n_txt, out_f32=out_f32, k_rotated=True,
                               v_f16=True)
    else:
        out, lse = dit.forward(qd, kd, vd, cs[0], cs[1], n_txt=w.n_txt, out_f32=out_f32)
    torch.cuda.synchronize()
    assert dit.dit_attn_get_status() == dit.DIT_OK
    return out, lse


def oracle_rows(w, q, k, v, rows, rope=True, operands="exact"):
    """operands="exact": rotation and attention in fp64 on the bf16 inputs.
    operands="bf16": rotated with the fp32 table entries and rounded to bf16,
    the precision the kernel's tensor cores take the rotated q, k in."""
    pos = W.positions(w) if rope else None
    if operands == "exact":
        return oracle_attention.joint_attention(q, k, v, pos=pos, rows=rows)
    return oracle_attention.joint_attention(q, k, v, pos=pos, rows=rows, round_rotated="bf16", table_fp32=True)


def near_midpoint_blocks(n_scales: int = 160, seed: int = 21):
    """bf16 values [1, 1, 64 * n_scales, 128] whose fp32 quotients by their
    block's scale land on or within a few ulps of an E4M3 rounding midpoint
    (where a quotient formed by multiplying with a rounded reciprocal can
    differ from the correctly rounded one).  Block b holds one element equal
    to its amax (scale = amax / 448 in fp32), then the bf16 values below amax
    whose quotients lie nearest to midpoints, then zeros.  Every third block
    has a power-of-two scale, so its quotients hit midpoints exactly (ties)."""
    rng = np.random.default_rng(seed)
    e4 = np.unique(np.abs(formats.e4m3_decode(np.arange(0x7F, dtype=np.uint8))))
    mids = ((e4[:-1] + e4[1:]) / 2).astype(np.float32)
    mid_bits = mids.view(np.uint32).astype(np.int64)
    # every positive finite bf16 value, as fp32
    all_bf16 = (np.arange(1, 0x7F80, dtype=np.uint32) << 16).view(np.float32)
    x = np.zeros((n_scales * 64, 128), np.float32)
    for b in range(n_scales):
        if b % 3 == 0:
            amax = np.float32(448.0 * 2.0 ** int(rng.integers(-12, 12)))
        else:
            amax = formats.round_bf16(np.float32(rng.uniform(0.05, 3000.0))).astype(np.float32)
        scale = np.float32(amax / np.float32(448.0))
        cand = all_bf16[all_bf16 < amax]
        q = (cand / scale).astype(np.float32)
        qb = q.view(np.uint32).astype(np.int64)
        i = np.clip(np.searchsorted(mid_bits, qb), 1, len(mid_bits) - 1)
        dist = np.minimum(np.abs(qb - mid_bits[i - 1]), np.abs(qb - mid_bits[i]))
        pick = cand[np.argsort(dist, kind="stable")[:64 * 128 - 1]]
        pick = pick * rng.choice(np.array([-1.0, 1.0], np.float32), pick.size)
        blk = np.zeros(64 * 128, np.float32)
        blk[0] = amax
        blk[1:1 + pick.size] = pick
        x[64 * b:64 * (b + 1)] = blk.reshape(64, 128)
    return x.reshape(1, 1, n_scales * 64, 128)
