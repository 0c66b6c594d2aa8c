"""The C ABI: the library loads, exports every entry point include/dit_attn.h
declares, and rejects bad arguments on the host before touching a GPU.  CPU only."""
import ctypes
import os
import re

import pytest

import diffusion_transformer_joint_attn_b200 as dit
from diffusion_transformer_joint_attn_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load_library()


def declared_functions():
    names = []
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(dit_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "dit_attn_forward" in names and "dit_rope_table_build" in names
    for n in names:
        assert hasattr(lib, n), n
    # the binding knows each of them too
    assert set(names) == set(_lib.SIGNATURES)


def test_status_strings(lib):
    assert dit.dit_attn_status_string(0) == "ok"
    assert "timed out" in dit.dit_attn_status_string(-5)
    assert dit.dit_attn_status_string(12345) == "unknown status"
    # no CUDA call has failed in this process: no recorded runtime error
    assert lib.dit_attn_last_cuda_error() == 0
    assert lib.dit_attn_last_cuda_error_string() == b"no error"


def _fwd(lib, q=0x10000, k=0x20000, v=0x30000, cos=None, sin=None, out=0x40000, lse=None, B=1, H=1, nt=8, ni=8, D=128,
         dtype=0):
    return lib.dit_attn_forward(q, k, v, cos, sin, out, lse, B, H, nt, ni, D, dtype, None)


def test_forward_argument_errors(lib):
    # every case below fails validation before any CUDA call
    assert _fwd(lib, q=None) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, out=None) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, cos=0x50000) == dit.DIT_ERR_INVALID_ARG          # sin missing
    assert _fwd(lib, B=0) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, H=-1) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, nt=0, ni=0) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, nt=-3) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, nt=2 ** 31 - 1, ni=2) == dit.DIT_ERR_INVALID_ARG
    assert _fwd(lib, D=64) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=dit.DIT_FP8_E4M3) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=0x800) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=dit.DIT_K_ROTATED) == dit.DIT_ERR_INVALID_ARG      # flag without tables
    assert _fwd(lib, q=0x10008) == dit.DIT_ERR_MISALIGNED
    assert _fwd(lib, out=0x40004) == dit.DIT_ERR_MISALIGNED
    assert _fwd(lib, cos=0x50000, sin=0x60008) == dit.DIT_ERR_MISALIGNED
    assert _fwd(lib, lse=0x70002) == dit.DIT_ERR_MISALIGNED


def test_split_form_argument_errors(lib):
    split = dit.DIT_QK_SPLIT
    assert _fwd(lib, dtype=split) == dit.DIT_ERR_INVALID_ARG                       # v must be the fp16 operand
    assert _fwd(lib, dtype=split | dit.DIT_V_F16 | dit.DIT_K_ROTATED) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=split | dit.DIT_V_F16 | dit.DIT_FP8_E4M3) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=split | dit.DIT_V_F16, D=64) == dit.DIT_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=split | dit.DIT_V_F16, k=0x20004) == dit.DIT_ERR_MISALIGNED
    # no block-sparse split form
    assert lib.dit_attn_forward_sparse(0x10000, 0x20000, 0x30000, None, None, 0x9000, 0x40000, None, 1, 1, 8, 8, 128,
                                       split | dit.DIT_V_F16, None) == dit.DIT_ERR_UNSUPPORTED
    f = lib.dit_attn_prepare_kv_split
    ok = dict(k=0x1000, v=0x2000, c=0x3000, s=0x4000, ks=0x5000, vf=0x6000, B=1, H=1, N=8, D=128)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["k"], a["v"], a["c"], a["s"], a["ks"], a["vf"], a["B"], a["H"], a["N"], a["D"], None)
    assert call(k=None) == dit.DIT_ERR_INVALID_ARG
    assert call(ks=None) == dit.DIT_ERR_INVALID_ARG
    assert call(s=None) == dit.DIT_ERR_INVALID_ARG                                 # cos without sin
    assert call(N=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(ks=0x5008) == dit.DIT_ERR_MISALIGNED
    assert call(c=0x3004) == dit.DIT_ERR_MISALIGNED


def test_key_set_forward_argument_errors(lib):
    f = lib.dit_attn_forward_kv

    def call(q=0x10000, k=0x20000, cos=None, sin=None, Nq=8, Nkv=16, D=128, dtype=0, lse=None):
        return f(q, k, 0x30000, cos, sin, 0x40000, lse, 1, 2, Nq, Nkv, D, dtype, None)
    assert call(q=None) == dit.DIT_ERR_INVALID_ARG
    assert call(Nq=0) == dit.DIT_ERR_INVALID_ARG
    assert call(Nkv=0) == dit.DIT_ERR_INVALID_ARG
    assert call(Nkv=-5) == dit.DIT_ERR_INVALID_ARG
    assert call(cos=0x50000) == dit.DIT_ERR_INVALID_ARG                            # sin missing
    # the tables rotate q only: k must come rotated (or split)
    assert call(cos=0x50000, sin=0x60000) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=0x800) == dit.DIT_ERR_UNSUPPORTED
    assert call(q=0x10008) == dit.DIT_ERR_MISALIGNED
    assert call(lse=0x70002) == dit.DIT_ERR_MISALIGNED
    assert call(cos=0x50000, sin=0x60000, dtype=dit.DIT_QK_SPLIT) == dit.DIT_ERR_INVALID_ARG   # v fp16 required


def test_projection_argument_errors(lib):
    f = lib.dit_qkv_project_fp8
    ok = dict(x=0x10000, w=0x20000, bias=None, c=None, s=None, q8=0x30000, k8=0x40000, v8=0x50000, qs=0x60000,
              ks=0x70000, vs=0x80000, q16=None, k16=None, v16=None, B=1, N=64, C=128, H=2, D=128)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["x"], a["w"], a["bias"], a["c"], a["s"], a["q8"], a["k8"], a["v8"], a["qs"], a["ks"], a["vs"],
                 a["q16"], a["k16"], a["v16"], a["B"], a["N"], a["C"], a["H"], a["D"], None)
    assert call(x=None) == dit.DIT_ERR_INVALID_ARG
    assert call(vs=None) == dit.DIT_ERR_INVALID_ARG
    assert call(c=0x90000) == dit.DIT_ERR_INVALID_ARG          # sin missing
    assert call(N=0) == dit.DIT_ERR_INVALID_ARG
    assert call(C=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(H=3) == dit.DIT_ERR_UNSUPPORTED                 # two heads per tile
    assert call(C=100) == dit.DIT_ERR_UNSUPPORTED               # rows of x and w 16-byte aligned
    assert call(x=0x10008) == dit.DIT_ERR_MISALIGNED
    assert call(q8=0x30004) == dit.DIT_ERR_MISALIGNED
    assert call(bias=0x90002) == dit.DIT_ERR_MISALIGNED
    assert call(k16=0xA0008) == dit.DIT_ERR_MISALIGNED


def test_sparse_forward_argument_errors(lib):
    f = lib.dit_attn_forward_sparse

    def call(mask=0x9000, nt=8, ni=8, q=0x10000, D=128, dtype=0):
        return f(q, 0x20000, 0x30000, None, None, mask, 0x40000, None, 1, 1, nt, ni, D, dtype, None)
    assert call(mask=None) == dit.DIT_ERR_INVALID_ARG
    assert call(nt=0, ni=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_FP8_E4M3) == dit.DIT_ERR_UNSUPPORTED
    assert call(nt=0, ni=dit.DIT_SPARSE_MAX_KV_TILES * 128 + 1) == dit.DIT_ERR_UNSUPPORTED
    assert call(q=0x10008) == dit.DIT_ERR_MISALIGNED


def test_host_forward_workspace_and_argument_errors(lib):
    f = lib.dit_attn_forward_host_workspace
    al = lambda x: (x + 255) // 256 * 256
    N = 1000
    one = 5 * al(4 * N * 128 * 2) + al(4 * N * 128 * 2) + al(4 * N * 4)      # q k v k_rot v16, bf16 out, lse
    assert f(1, 24, N, 128, 0, 4) == 3 * one                               # three buffers
    assert f(1, 2, N, 128, 0, 4) == 3 * (5 * al(2 * N * 256) + al(2 * N * 256) + al(2 * N * 4))   # chunk <= B*H
    assert f(1, 24, N, 128, dit.DIT_OUT_F32, 4) == 3 * (one - al(4 * N * 256) + al(4 * N * 512))
    assert f(1, 24, N, 64, 0, 4) == 0 and f(1, 24, N, 128, 0, 0) == 0 and f(1, 24, N, 128, 1, 4) == 0
    g = lib.dit_attn_forward_host
    ok = dict(q=0x1000, ws=0x8000, wsb=3 * one, chunk=4, D=128, dtype=0)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["q"], 0x2000, 0x3000, None, None, 0x4000, None, 1, 24, 0, N, a["D"], a["dtype"], a["ws"], a["wsb"],
                 a["chunk"], None)
    assert call(q=None) == dit.DIT_ERR_INVALID_ARG
    assert call(ws=None) == dit.DIT_ERR_INVALID_ARG
    assert call(wsb=3 * one - 1) == dit.DIT_ERR_INVALID_ARG
    assert call(chunk=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_K_ROTATED) == dit.DIT_ERR_UNSUPPORTED
    assert call(ws=0x8008) == dit.DIT_ERR_MISALIGNED


def test_static_workspace_entry_rejects_oversize_without_a_gpu(lib):
    # the size check comes before any CUDA call: 2048x2048 in 4-head chunks needs ~312 MB of workspace
    rc = lib.dit_attn_forward_host_static(0x1000, 0x2000, 0x3000, None, None, 0x4000, None, 1, 24, 512, 16384, 128,
                                          0, 4, None)
    assert rc == dit.DIT_ERR_WORKSPACE
    assert dit.dit_attn_status_string(rc) == "problem needs more workspace than the static workspace holds"


def test_static_workspace_token_limit_at_one_head_per_chunk(lib):
    """The header's largest N for the static workspace holds at chunk_heads = 1,
    the smallest chunk: N fits, N + 1 does not (bf16 and fp32 output)."""
    size = lib.dit_attn_forward_host_workspace
    for dtype, n_max in ((dit.DIT_BF16, 7262), (dit.DIT_BF16 | dit.DIT_OUT_F32, 6227)):
        assert size(1, 1, n_max, 128, dtype, 1) <= 32 << 20
        assert size(1, 1, n_max + 1, 128, dtype, 1) > 32 << 20
        # one head per chunk is the minimum whatever chunk_heads asks for
        assert size(1, 24, n_max + 1, 128, dtype, 1) > 32 << 20
        rc = lib.dit_attn_forward_host_static(0x1000, 0x2000, 0x3000, None, None, 0x4000, None, 1, 24, 0,
                                              n_max + 1, 128, dtype, 1, None)
        assert rc == dit.DIT_ERR_WORKSPACE


def test_static_workspace_entry_argument_errors_before_any_cuda_call(lib):
    f = lib.dit_attn_forward_host_static

    def call(q=0x1000, B=1, H=2, nt=16, ni=48, D=128, dtype=0, chunk=1, cos=None, sin=None):
        return f(q, 0x2000, 0x3000, cos, sin, 0x4000, None, B, H, nt, ni, D, dtype, chunk, None)
    assert call(q=None) == dit.DIT_ERR_INVALID_ARG
    assert call(cos=0x5000) == dit.DIT_ERR_INVALID_ARG                    # sin missing
    assert call(B=0) == dit.DIT_ERR_INVALID_ARG
    assert call(nt=0, ni=0) == dit.DIT_ERR_INVALID_ARG
    assert call(chunk=0) == dit.DIT_ERR_INVALID_ARG
    assert call(B=65536, H=65536) == dit.DIT_ERR_INVALID_ARG             # B * H beyond int
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_V_F16) == dit.DIT_ERR_UNSUPPORTED


def test_host_entries_reject_head_counts_beyond_int(lib):
    assert lib.dit_attn_forward_host_workspace(65536, 65536, 16, 128, 0, 4) == 0
    rc = lib.dit_attn_forward_host(0x1000, 0x2000, 0x3000, None, None, 0x4000, None, 65536, 65536, 0, 16, 128, 0,
                                   0x8000, 1 << 40, 4, None)
    assert rc == dit.DIT_ERR_INVALID_ARG


def test_rope_table_argument_errors(lib):
    ax = (ctypes.c_int32 * 3)(16, 56, 56)
    bad = (ctypes.c_int32 * 3)(16, 55, 57)
    short = (ctypes.c_int32 * 3)(16, 56, 50)
    f = lib.dit_rope_table_build
    assert f(None, 8, 128, ax, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x100, 0, 128, ax, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x100, 8, 128, ax, 0.0, 0x1000, 0x2000, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x100, 8, 128, bad, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x100, 8, 128, short, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x100, 8, 96, ax, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_UNSUPPORTED
    assert f(0x102, 8, 128, ax, 1e4, 0x1000, 0x2000, None) == dit.DIT_ERR_MISALIGNED
    assert f(0x100, 8, 128, ax, 1e4, 0x1004, 0x2000, None) == dit.DIT_ERR_MISALIGNED


def test_operand_pass_argument_errors(lib):
    f = lib.dit_attn_prepare_kv
    ok = dict(k=0x1000, v=0x2000, c=0x3000, s=0x4000, kr=0x5000, vf=0x6000, B=1, H=1, N=8, D=128)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["k"], a["v"], a["c"], a["s"], a["kr"], a["vf"], a["B"], a["H"], a["N"], a["D"], None)
    assert call(k=None) == dit.DIT_ERR_INVALID_ARG
    assert call(vf=None) == dit.DIT_ERR_INVALID_ARG
    assert call(N=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(v=0x2008) == dit.DIT_ERR_MISALIGNED
    g = lib.dit_rope_apply
    assert g(None, 0x3000, 0x4000, 0x5000, 1, 1, 8, 128, None) == dit.DIT_ERR_INVALID_ARG
    assert g(0x1000, 0x3000, 0x4000, 0x5000, 1, 1, 8, 64, None) == dit.DIT_ERR_UNSUPPORTED
    assert g(0x1004, 0x3000, 0x4000, 0x5000, 1, 1, 8, 128, None) == dit.DIT_ERR_MISALIGNED


def test_fp8_argument_errors(lib):
    f = lib.dit_attn_quantize_fp8
    assert f(None, None, None, 0x2000, 0x3000, 1, 1, 8, 128, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x1000, 0x4000, None, 0x2000, 0x3000, 1, 1, 8, 128, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x1000, None, None, 0x2000, 0x3000, 1, 1, 0, 128, None) == dit.DIT_ERR_INVALID_ARG
    assert f(0x1000, None, None, 0x2000, 0x3000, 1, 1, 8, 64, None) == dit.DIT_ERR_UNSUPPORTED
    assert f(0x1000, None, None, 0x2008, 0x3000, 1, 1, 8, 128, None) == dit.DIT_ERR_MISALIGNED
    assert f(0x1000, None, None, 0x2000, 0x3002, 1, 1, 8, 128, None) == dit.DIT_ERR_MISALIGNED
    g = lib.dit_attn_forward_fp8
    ok = dict(q=0x1000, k=0x2000, v=0x3000, qs=0x4000, ks=0x5000, vs=0x6000, out=0x7000, lse=None, B=1, H=1,
              nt=8, ni=8, D=128, dtype=dit.DIT_FP8_E4M3)

    def call(**kw):
        a = dict(ok, **kw)
        return g(a["q"], a["k"], a["v"], a["qs"], a["ks"], a["vs"], a["out"], a["lse"], a["B"], a["H"], a["nt"],
                 a["ni"], a["D"], a["dtype"], None)
    assert call(v=None) == dit.DIT_ERR_INVALID_ARG
    assert call(ks=None) == dit.DIT_ERR_INVALID_ARG
    assert call(nt=0, ni=0) == dit.DIT_ERR_INVALID_ARG
    assert call(B=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_BF16) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_FP8_E4M3 | dit.DIT_K_ROTATED) == dit.DIT_ERR_UNSUPPORTED
    assert call(q=0x1001) == dit.DIT_ERR_MISALIGNED
    assert call(vs=0x6002) == dit.DIT_ERR_MISALIGNED
    assert call(lse=0x8001) == dit.DIT_ERR_MISALIGNED


def test_merge_argument_errors(lib):
    f = lib.dit_attn_merge

    def call(R=2, o=(0x1000, 0x2000), l=(0x3000, 0x4000), out=0x5000, lse=None, B=1, H=1, N=8, D=128, dtype=0):
        oa = (ctypes.c_void_p * max(len(o), 1))(*o)
        la = (ctypes.c_void_p * max(len(l), 1))(*l)
        return f(ctypes.cast(oa, ctypes.c_void_p), ctypes.cast(la, ctypes.c_void_p), R, out, lse, B, H, N, D, dtype,
                 None)
    assert f(None, None, 1, 0x5000, None, 1, 1, 8, 128, 0, None) == dit.DIT_ERR_INVALID_ARG
    assert call(R=0) == dit.DIT_ERR_INVALID_ARG
    assert call(R=17, o=(0x1000,) * 17, l=(0x3000,) * 17) == dit.DIT_ERR_INVALID_ARG
    assert call(o=(0x1000, None)) == dit.DIT_ERR_INVALID_ARG
    assert call(out=None) == dit.DIT_ERR_INVALID_ARG
    assert call(N=0) == dit.DIT_ERR_INVALID_ARG
    assert call(D=64) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_FP8_E4M3) == dit.DIT_ERR_UNSUPPORTED
    assert call(dtype=dit.DIT_K_ROTATED) == dit.DIT_ERR_UNSUPPORTED
    assert call(o=(0x1000, 0x2008)) == dit.DIT_ERR_MISALIGNED
    assert call(l=(0x3000, 0x4002)) == dit.DIT_ERR_MISALIGNED
    assert call(lse=0x6001) == dit.DIT_ERR_MISALIGNED


def test_wait_selftest_limit_range(lib):
    assert lib.dit_attn_wait_selftest(999, None) == dit.DIT_ERR_INVALID_ARG
    assert lib.dit_attn_wait_selftest(2 * 10 ** 9, None) == dit.DIT_ERR_INVALID_ARG


def test_get_status_rejects_null(lib):
    assert lib.dit_attn_get_status(None, None) == dit.DIT_ERR_INVALID_ARG


def test_binding_refuses_cuda_tensors_on_several_devices():
    import torch

    class OnDevice:                      # the two attributes the check reads of a CUDA tensor
        def __init__(self, index):
            self.is_cuda = True
            self.device = torch.device("cuda", index)
    with pytest.raises(ValueError, match="one device"):
        dit._on_current_device(OnDevice(0), None, OnDevice(1))
    dit._on_current_device(None, torch.zeros(2))     # no CUDA tensor: nothing to check, no CUDA call


def test_binding_marshalling_errors():
    import torch
    q = torch.zeros(1, 1, 4, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dit.dit_attn_forward(q, q, q, None, None, q, None, 2, 2)      # CPU tensors are refused
