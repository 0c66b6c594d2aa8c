"""dit_attn_forward_host_static, the entry point that allocates nothing (its
workspace is a static array of the library), against dit_attn_forward_host
with a caller workspace.  Needs a B200.

Collected last on purpose: it must also pass after every other test has run
in the same process, as well as alone in a fresh one.  The same kernels run
on the same values, so the results are compared bit for bit (tighter than
the BF16 parity bars)."""
import ctypes

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


def static_call(lib, w, q, k, v, c, s, chunk_heads):
    out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=True)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.current_stream()
    rc = lib.dit_attn_forward_host_static(q.data_ptr(), k.data_ptr(), v.data_ptr(), c.data_ptr(), s.data_ptr(),
                                          out.data_ptr(), lse.data_ptr(), w.B, w.H, w.n_txt, w.n_img, w.D,
                                          dit.DIT_BF16, chunk_heads, ctypes.c_void_p(stream.cuda_stream))
    stream.synchronize()
    return rc, out, lse


def test_static_workspace_entry_matches_caller_workspace_entry():
    lib = dit.load_library()
    w = W.WORKLOADS["t2i_512px"]                   # B=1, H=24, N=1536: 4-head chunks fit in the static array
    q, k, v = (t.pin_memory() for t in W.make_qkv(w, seed=5))
    c, s = dit.rope_table(torch.from_numpy(W.positions(w)).cuda())
    chunk = 4
    assert dit.dit_attn_forward_host_workspace(w.B, w.H, w.N, dit.DIT_BF16, chunk) <= dit.DIT_STATIC_WORKSPACE_BYTES
    ref, lref = dit.forward_host(q, k, v, c, s, n_txt=w.n_txt, chunk_heads=chunk)
    for _ in range(2):                             # twice in a row: the array is reused
        rc, out, lse = static_call(lib, w, q, k, v, c, s, chunk)
        assert rc == dit.DIT_OK, dit.dit_attn_status_string(rc)
        assert torch.equal(out, ref) and torch.equal(lse, lref)
    assert dit.dit_attn_get_status() == dit.DIT_OK


def test_static_workspace_entry_rejects_what_does_not_fit():
    lib = dit.load_library()
    w = W.WORKLOADS["t2i_2048px"]                  # N = 16896: 4-head chunks need about 312 MB
    assert dit.dit_attn_forward_host_workspace(w.B, w.H, w.N, dit.DIT_BF16, 4) > dit.DIT_STATIC_WORKSPACE_BYTES
    q = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.bfloat16)
    rc = lib.dit_attn_forward_host_static(q.data_ptr(), q.data_ptr(), q.data_ptr(), None, None, q.data_ptr(), None,
                                          w.B, w.H, w.n_txt, w.n_img, w.D, dit.DIT_BF16, 4, None)
    assert rc == dit.DIT_ERR_WORKSPACE
    assert "static workspace" in dit.dit_attn_status_string(rc)
