"""dit_attn_forward_host (q, k, v and the results in host memory, copies
overlapped with the kernels) against the device-memory forward.  Needs a
B200.  The same kernels run on the same values, so the results must be equal
bit for bit, whatever the chunking, pinning or workspace reuse."""
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit
import workloads as W
from diffusion_transformer_joint_attn_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    dit.load_library()


def device_reference(w, q, k, v, rope=True, out_f32=False):
    c, s = dit.rope_table(torch.from_numpy(W.positions(w)).cuda()) if rope else (None, None)
    out, lse = dit.forward(q.cuda(), k.cuda(), v.cuda(), c, s, n_txt=w.n_txt, out_f32=out_f32)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu(), c, s


@pytest.mark.parametrize("chunk_heads", [1, 5, 48])
def test_host_forward_equals_device_forward(chunk_heads):
    w = W.WORKLOADS["t2i_1024px_cfg"]              # B*H = 48 (head pairs), N = 4608
    q, k, v = W.make_qkv(w, seed=2)
    ref, lref, c, s = device_reference(w, q, k, v)
    out, lse = dit.forward_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), c, s, n_txt=w.n_txt,
                                chunk_heads=chunk_heads)
    assert torch.equal(out, ref) and torch.equal(lse, lref)


def test_pageable_memory_fp32_output_and_no_rope():
    w = W.custom(1, 3, 40, ((10, 12),))
    q, k, v = W.make_qkv(w, seed=3)
    ref, lref, c, s = device_reference(w, q, k, v, out_f32=True)
    out, lse = dit.forward_host(q, k, v, c, s, n_txt=w.n_txt, out_f32=True, chunk_heads=2, pin=False)
    assert torch.equal(out, ref) and torch.equal(lse, lref)
    ref2, lref2, _, _ = device_reference(w, q, k, v, rope=False)
    out2, lse2 = dit.forward_host(q, k, v, n_txt=w.n_txt, chunk_heads=2)
    assert torch.equal(out2, ref2) and torch.equal(lse2, lref2)


def test_workspace_reuse_across_calls_without_sync():
    """Back-to-back calls on one workspace and stream, synchronised once at
    the end: the library orders the reuse of its buffers."""
    w = W.custom(2, 3, 64, ((16, 16),))
    c, s = dit.rope_table(torch.from_numpy(W.positions(w)).cuda())
    nbytes = dit.dit_attn_forward_host_workspace(w.B, w.H, w.N, dit.DIT_BF16, 2)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    results = []
    for seed in range(4):
        q, k, v = (t.pin_memory() for t in W.make_qkv(w, seed=seed))
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, pin_memory=True)
        dit.dit_attn_forward_host(q, k, v, c, s, out, lse, w.n_txt, w.n_img, ws, chunk_heads=2)
        results.append((q, k, v, out, lse))
    torch.cuda.synchronize()
    for q, k, v, out, lse in results:
        ref, lref, _, _ = device_reference(w, q, k, v)
        assert torch.equal(out, ref) and torch.equal(lse, lref)
    assert dit.dit_attn_get_status() == dit.DIT_OK
