"""Python binding of libdit_attn, the B200 joint text+image attention library.

Argument marshalling only: every function below hands raw device pointers,
sizes and the stream to the C entry point of the same name (declared in
include/dit_attn.h).  Torch tensors serve as device buffers; all computation
happens in the library's CUDA kernels.  There is no fallback: if the shared
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

from ._lib import load_library, library_path  # noqa: F401

DIT_OK = 0
DIT_ERR_INVALID_ARG = -1
DIT_ERR_UNSUPPORTED = -2
DIT_ERR_MISALIGNED = -3
DIT_ERR_CUDA = -4
DIT_ERR_TIMEOUT = -5
DIT_ERR_WORKSPACE = -6
DIT_STATIC_WORKSPACE_BYTES = 32 << 20
DIT_BF16 = 0
DIT_FP8_E4M3 = 1
DIT_OUT_F32 = 0x100
DIT_K_ROTATED = 0x200
DIT_V_F16 = 0x400
DIT_PART_F32 = 0x800
DIT_QK_SPLIT = 0x1000
DIT_MERGE_MAX_PARTS = 16
DIT_SPARSE_MAX_KV_TILES = 4096


class DitError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = "%s failed: %s (%d)" % (what, dit_attn_status_string(status), status)
        if status == DIT_ERR_CUDA:
            lib = load_library()
            msg += ": %s (%d)" % (lib.dit_attn_last_cuda_error_string().decode(), lib.dit_attn_last_cuda_error())
        super().__init__(msg)


def _check(status: int, what: str) -> None:
    if status != DIT_OK:
        raise DitError(status, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _require(cond: bool, msg: str) -> None:
    if not cond:
        raise ValueError(msg)


def _on_current_device(*tensors) -> None:
    """The library launches on the current CUDA device and hands it the
    tensors' addresses, so every CUDA tensor of a call (None entries are
    skipped) must live on that one device; anything else is refused here
    instead of reaching a kernel as another device's address."""
    devs = {t.device for t in tensors if t is not None and t.is_cuda}
    _require(len(devs) <= 1, "the CUDA tensors of one call must be on one device, not %s" %
             ", ".join(sorted(str(d) for d in devs)))
    if devs:
        import torch
        dev = devs.pop()
        cur = torch.cuda.current_device()
        _require(dev.index == cur, "the tensors are on %s but the current device is cuda:%d "
                 "(torch.cuda.set_device selects it)" % (dev, cur))


def dit_rope_table_build(pos, axes: Sequence[int], theta: float, rope_cos, rope_sin, stream=None) -> None:
    """Fill rope_cos / rope_sin (CUDA fp32 [N, 64]) from positions pos (CUDA int32 [N, 3])."""
    import torch
    _require(pos.is_cuda and pos.dtype == torch.int32 and pos.dim() == 2 and pos.shape[1] == 3 and
             pos.is_contiguous(), "pos must be a contiguous CUDA int32 [N, 3] tensor")
    N = pos.shape[0]
    for t in (rope_cos, rope_sin):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (N, 64),
                 "rope tables must be contiguous CUDA fp32 [N, 64] tensors")
    _on_current_device(pos, rope_cos, rope_sin)
    ax = (ctypes.c_int32 * 3)(*[int(a) for a in axes])
    _check(load_library().dit_rope_table_build(_ptr(pos), N, 128, ax, float(theta), _ptr(rope_cos),
                                               _ptr(rope_sin), _stream(stream)), "dit_rope_table_build")


def dit_rope_apply(x, rope_cos, rope_sin, x_rot, stream=None) -> None:
    """x_rot <- rotary embedding of bf16 x [B, H, N, D] (x_rot may be x)."""
    import torch
    _require(x.dim() == 4 and x.shape == x_rot.shape, "x and x_rot must share one [B, H, N, D] shape")
    B, H, N, D = x.shape
    for t in (x, x_rot):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "x, x_rot must be contiguous CUDA bf16")
    for t in (rope_cos, rope_sin):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (N, D // 2),
                 "rope tables must be contiguous CUDA fp32 [N, D/2]")
    _on_current_device(x, rope_cos, rope_sin, x_rot)
    _check(load_library().dit_rope_apply(_ptr(x), _ptr(rope_cos), _ptr(rope_sin), _ptr(x_rot), B, H, N, D,
                                         _stream(stream)), "dit_rope_apply")


def dit_attn_prepare_kv(k, v, rope_cos, rope_sin, k_rot, v_f16, stream=None) -> None:
    """k_rot <- rotated bf16 k, v_f16 <- fp16 copy of v (both [B, H, N, D])."""
    import torch
    _require(k.dim() == 4 and k.shape == v.shape == k_rot.shape == v_f16.shape, "k, v, k_rot, v_f16 shapes differ")
    B, H, N, D = k.shape
    for t in (k, v, k_rot):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "k, v, k_rot must be contiguous CUDA bf16")
    _require(v_f16.is_cuda and v_f16.dtype == torch.float16 and v_f16.is_contiguous(), "v_f16 must be CUDA fp16")
    for t in (rope_cos, rope_sin):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and tuple(t.shape) == (N, D // 2),
                 "rope tables must be contiguous CUDA fp32 [N, D/2]")
    _on_current_device(k, v, rope_cos, rope_sin, k_rot, v_f16)
    _check(load_library().dit_attn_prepare_kv(_ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), _ptr(k_rot),
                                              _ptr(v_f16), B, H, N, D, _stream(stream)), "dit_attn_prepare_kv")


def dit_attn_prepare_kv_split(k, v, rope_cos, rope_sin, k_split, v_f16, stream=None) -> None:
    """k_split <- fp16 [2, B, H, N, D] hi / lo split of the rotated k, v_f16 <- fp16 copy of v; the tables may
    both be None (no rotation)."""
    import torch
    _require(k.dim() == 4 and k.shape == v.shape == v_f16.shape, "k, v, v_f16 shapes differ")
    B, H, N, D = k.shape
    _require(tuple(k_split.shape) == (2, B, H, N, D), "k_split must be [2, B, H, N, D]")
    for t in (k, v):
        _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "k, v must be contiguous CUDA bf16")
    for t in (k_split, v_f16):
        _require(t.is_cuda and t.dtype == torch.float16 and t.is_contiguous(), "k_split, v_f16 must be CUDA fp16")
    _check_tables(rope_cos, rope_sin, N, D)
    _on_current_device(k, v, rope_cos, rope_sin, k_split, v_f16)
    _check(load_library().dit_attn_prepare_kv_split(_ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), _ptr(k_split),
                                                    _ptr(v_f16), B, H, N, D, _stream(stream)),
           "dit_attn_prepare_kv_split")


def _check_tables(rope_cos, rope_sin, N, D):
    """Both tables None, or both contiguous CUDA fp32 [N, D/2]."""
    import torch
    if rope_cos is not None or rope_sin is not None:
        for t in (rope_cos, rope_sin):
            _require(t is not None and t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (N, D // 2), "rope tables must be contiguous CUDA fp32 [N, D/2]")


def dit_attn_forward_kv(q, k, v, q_cos, q_sin, out, lse, dtype: int = DIT_BF16, stream=None) -> None:
    """out (and lse) <- attention of bf16 q [B, H, N_q, D] to the N_kv keys and values k, v [B, H, N_kv, D]
    (k: the [2, B, H, N_kv, D] fp16 split operand with DIT_QK_SPLIT); q_cos / q_sin: the queries' table rows."""
    import torch
    _require(q.dim() == 4 and v.dim() == 4 and q.shape[:2] == v.shape[:2] and q.shape[3] == v.shape[3],
             "q [B, H, N_q, D] and v [B, H, N_kv, D] must agree in B, H, D")
    B, H, N_q, D = q.shape
    N_kv = v.shape[2]
    _check_operands(q, k, v, out, lse, dtype, N_kv)
    _check_tables(q_cos, q_sin, N_q, D)
    _on_current_device(q, k, v, q_cos, q_sin, out, lse)
    _check(load_library().dit_attn_forward_kv(_ptr(q), _ptr(k), _ptr(v), _ptr(q_cos), _ptr(q_sin), _ptr(out),
                                              _ptr(lse), B, H, N_q, N_kv, D, dtype, _stream(stream)),
           "dit_attn_forward_kv")


def _check_operands(q, k, v, out, lse, dtype, N_kv):
    """dtype / shape checks of q, k, v, out, lse for N_q queries (q.shape[2]) and N_kv keys."""
    import torch
    B, H, N_q, D = q.shape
    _require(q.is_cuda and q.dtype == torch.bfloat16 and q.is_contiguous(), "q must be contiguous CUDA bf16")
    if dtype & DIT_QK_SPLIT:
        _require(tuple(k.shape) == (2, B, H, N_kv, D) and k.is_cuda and k.dtype == torch.float16 and
                 k.is_contiguous(), "with DIT_QK_SPLIT, k must be the contiguous CUDA fp16 [2, B, H, N_kv, D] "
                 "operand of dit_attn_prepare_kv_split")
    else:
        _require(tuple(k.shape) == (B, H, N_kv, D) and k.is_cuda and k.dtype == torch.bfloat16 and k.is_contiguous(),
                 "k must be a contiguous CUDA bf16 [B, H, N_kv, D] tensor")
    v_dtype = torch.float16 if dtype & DIT_V_F16 else torch.bfloat16
    _require(tuple(v.shape) == (B, H, N_kv, D) and v.is_cuda and v.dtype == v_dtype and v.is_contiguous(),
             "v must be a contiguous CUDA bf16 (fp16 with DIT_V_F16) [B, H, N_kv, D] tensor")
    out_dtype = torch.float32 if dtype & DIT_OUT_F32 else torch.bfloat16
    _require(out.is_cuda and out.dtype == out_dtype and out.is_contiguous() and out.shape == q.shape,
             "out must be a contiguous CUDA tensor of q's shape and the requested dtype")
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and
                 tuple(lse.shape) == (B, H, N_q), "lse must be a contiguous CUDA fp32 [B, H, N_q] tensor")


def dit_attn_forward(q, k, v, rope_cos, rope_sin, out, lse, n_txt: int, n_img: int, dtype: int = DIT_BF16,
                     stream=None) -> None:
    """out (and lse, if not None) <- joint attention of bf16 q, k, v [B, H, N, D] on the GPU."""
    B, H, N, D = q.shape
    _check_forward_args(q, k, v, rope_cos, rope_sin, out, lse, n_txt, n_img, dtype)
    _check(load_library().dit_attn_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), _ptr(out),
                                           _ptr(lse), B, H, n_txt, n_img, D, dtype, _stream(stream)),
           "dit_attn_forward")


def _check_forward_args(q, k, v, rope_cos, rope_sin, out, lse, n_txt, n_img, dtype):
    _require(q.dim() == 4 and v.dim() == 4 and q.shape == v.shape, "q, k, v must share one [B, H, N, D] shape")
    B, H, N, D = q.shape
    _require(N == n_txt + n_img, "N must equal n_txt + n_img")
    _check_operands(q, k, v, out, lse, dtype, N)
    _check_tables(rope_cos, rope_sin, N, D)
    _on_current_device(q, k, v, rope_cos, rope_sin, out, lse)


def dit_attn_forward_host_workspace(B: int, H: int, N: int, dtype: int = DIT_BF16, chunk_heads: int = 4) -> int:
    """Device workspace bytes dit_attn_forward_host needs (0 for invalid arguments)."""
    return int(load_library().dit_attn_forward_host_workspace(B, H, N, 128, dtype, chunk_heads))


def dit_attn_forward_host(q, k, v, rope_cos, rope_sin, out, lse, n_txt: int, n_img: int, workspace,
                          dtype: int = DIT_BF16, chunk_heads: int = 4, stream=None) -> None:
    """out, lse (CPU tensors) <- joint attention of CPU bf16 q, k, v [B, H, N, D]; the tables and the
    workspace (uint8) are CUDA tensors.  Pinned CPU tensors let the copies overlap the kernels."""
    import torch
    _require(q.dim() == 4 and q.shape == k.shape == v.shape, "q, k, v must share one [B, H, N, D] shape")
    B, H, N, D = q.shape
    _require(N == n_txt + n_img, "N must equal n_txt + n_img")
    for t in (q, k, v):
        _require(not t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous(), "q, k, v must be contiguous CPU bf16")
    out_dtype = torch.float32 if dtype & DIT_OUT_F32 else torch.bfloat16
    _require(not out.is_cuda and out.dtype == out_dtype and out.is_contiguous() and out.shape == q.shape,
             "out must be a contiguous CPU tensor of q's shape and the requested dtype")
    if lse is not None:
        _require(not lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and
                 tuple(lse.shape) == (B, H, N), "lse must be a contiguous CPU fp32 [B, H, N] tensor")
    if rope_cos is not None or rope_sin is not None:
        for t in (rope_cos, rope_sin):
            _require(t is not None and t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (N, D // 2), "rope tables must be contiguous CUDA fp32 [N, D/2]")
    _require(workspace.is_cuda and workspace.is_contiguous(), "workspace must be a contiguous CUDA tensor")
    _on_current_device(rope_cos, rope_sin, workspace)
    nbytes = workspace.numel() * workspace.element_size()
    _check(load_library().dit_attn_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin), _ptr(out),
                                                _ptr(lse), B, H, n_txt, n_img, D, dtype, _ptr(workspace), nbytes,
                                                chunk_heads, _stream(stream)), "dit_attn_forward_host")


def dit_attn_forward_sparse(q, k, v, rope_cos, rope_sin, kv_mask, out, lse, n_txt: int, n_img: int,
                            dtype: int = DIT_BF16, stream=None) -> None:
    """dit_attn_forward restricted to the key tiles of kv_mask (CUDA uint8
    [B, H, ceil(N/512), ceil(N/128)], nonzero = attend)."""
    import torch
    B, H, N, D = q.shape
    _require(kv_mask is not None and kv_mask.is_cuda and kv_mask.dtype == torch.uint8 and kv_mask.is_contiguous()
             and tuple(kv_mask.shape) == (B, H, (N + 511) // 512, (N + 127) // 128),
             "kv_mask must be a contiguous CUDA uint8 [B, H, ceil(N/512), ceil(N/128)] tensor")
    _check_forward_args(q, k, v, rope_cos, rope_sin, out, lse, n_txt, n_img, dtype)
    _on_current_device(kv_mask)
    _check(load_library().dit_attn_forward_sparse(_ptr(q), _ptr(k), _ptr(v), _ptr(rope_cos), _ptr(rope_sin),
                                                  _ptr(kv_mask), _ptr(out), _ptr(lse), B, H, n_txt, n_img, D, dtype,
                                                  _stream(stream)), "dit_attn_forward_sparse")


def dit_attn_quantize_fp8(x, rope_cos, rope_sin, x_fp8, scale, stream=None) -> None:
    """x_fp8 (uint8 E4M3 codes) and scale (fp32 per 64-token block) of bf16 x [B, H, N, D]."""
    import torch
    _require(x.dim() == 4 and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous(), "x must be CUDA bf16")
    B, H, N, D = x.shape
    _require(x_fp8.is_cuda and x_fp8.dtype == torch.uint8 and x_fp8.is_contiguous() and x_fp8.shape == x.shape,
             "x_fp8 must be a contiguous CUDA uint8 tensor of x's shape")
    _require(scale.is_cuda and scale.dtype == torch.float32 and scale.is_contiguous() and
             tuple(scale.shape) == (B, H, (N + 63) // 64), "scale must be CUDA fp32 [B, H, ceil(N/64)]")
    if rope_cos is not None or rope_sin is not None:
        for t in (rope_cos, rope_sin):
            _require(t is not None and t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                     tuple(t.shape) == (N, D // 2), "rope tables must be contiguous CUDA fp32 [N, D/2]")
    _on_current_device(x, rope_cos, rope_sin, x_fp8, scale)
    _check(load_library().dit_attn_quantize_fp8(_ptr(x), _ptr(rope_cos), _ptr(rope_sin), _ptr(x_fp8), _ptr(scale),
                                                B, H, N, D, _stream(stream)), "dit_attn_quantize_fp8")


def quantize_fp8(x, rope_cos=None, rope_sin=None, stream=None):
    """Allocate and fill (codes, scales) for bf16 x [B, H, N, D]."""
    import torch
    B, H, N, D = x.shape
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    scale = torch.empty((B, H, (N + 63) // 64), dtype=torch.float32, device=x.device)
    dit_attn_quantize_fp8(x, rope_cos, rope_sin, codes, scale, stream)
    return codes, scale


def dit_attn_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, out, lse, n_txt: int, n_img: int,
                         dtype: int = DIT_FP8_E4M3, stream=None) -> None:
    """out (and lse, if not None) <- joint attention of E4M3 codes q8, k8, v8 [B, H, N, D] with
    per-64-token fp32 scales [B, H, ceil(N/64)]."""
    import torch
    _require(q8.dim() == 4 and q8.shape == k8.shape == v8.shape, "q8, k8, v8 must share one [B, H, N, D] shape")
    B, H, N, D = q8.shape
    _require(N == n_txt + n_img, "N must equal n_txt + n_img")
    for t in (q8, k8, v8):
        _require(t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous(), "q8, k8, v8 must be contiguous CUDA uint8")
    for t in (q_scale, k_scale, v_scale):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                 tuple(t.shape) == (B, H, (N + 63) // 64), "scales must be contiguous CUDA fp32 [B, H, ceil(N/64)]")
    out_dtype = torch.float32 if dtype & DIT_OUT_F32 else torch.bfloat16
    _require(out.is_cuda and out.dtype == out_dtype and out.is_contiguous() and out.shape == q8.shape,
             "out must be a contiguous CUDA tensor of q8's shape and the requested dtype")
    if lse is not None:
        _require(lse.is_cuda and lse.dtype == torch.float32 and lse.is_contiguous() and tuple(lse.shape) == (B, H, N),
                 "lse must be a contiguous CUDA fp32 [B, H, N] tensor")
    _on_current_device(q8, k8, v8, q_scale, k_scale, v_scale, out, lse)
    _check(load_library().dit_attn_forward_fp8(_ptr(q8), _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale),
                                               _ptr(v_scale), _ptr(out), _ptr(lse), B, H, n_txt, n_img, D, dtype,
                                               _stream(stream)), "dit_attn_forward_fp8")


def dit_qkv_project_fp8(x, w, bias, rope_cos, rope_sin, q8, k8, v8, q_scale, k_scale, v_scale, q16=None, k16=None,
                        v16=None, stream=None) -> None:
    """E4M3 codes and block scales of the rotated q, k and of v (and optionally the bf16 q, k, v) from the QKV
    projection of the hidden states x [B, N, C] (bf16) with the weight w [3 H 128, C] (bf16) and an optional fp32
    bias [3 H 128]."""
    import torch
    _require(x.dim() == 3 and x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous(),
             "x must be a contiguous CUDA bf16 [B, N, C] tensor")
    B, N, C = x.shape
    _require(w.dim() == 2 and w.shape[1] == C and w.shape[0] % 384 == 0 and w.is_cuda and w.dtype == torch.bfloat16
             and w.is_contiguous(), "w must be a contiguous CUDA bf16 [3 H 128, C] tensor")
    H = w.shape[0] // 384
    if bias is not None:
        _require(bias.is_cuda and bias.dtype == torch.float32 and bias.is_contiguous() and
                 tuple(bias.shape) == (w.shape[0],), "bias must be a contiguous CUDA fp32 [3 H 128] tensor")
    _check_tables(rope_cos, rope_sin, N, 128)
    for t in (q8, k8, v8):
        _require(t.is_cuda and t.dtype == torch.uint8 and t.is_contiguous() and tuple(t.shape) == (B, H, N, 128),
                 "q8, k8, v8 must be contiguous CUDA uint8 [B, H, N, 128] tensors")
    for t in (q_scale, k_scale, v_scale):
        _require(t.is_cuda and t.dtype == torch.float32 and t.is_contiguous() and
                 tuple(t.shape) == (B, H, (N + 63) // 64), "scales must be contiguous CUDA fp32 [B, H, ceil(N/64)]")
    for t in (q16, k16, v16):
        if t is not None:
            _require(t.is_cuda and t.dtype == torch.bfloat16 and t.is_contiguous() and
                     tuple(t.shape) == (B, H, N, 128), "q16, k16, v16 must be contiguous CUDA bf16 [B, H, N, 128]")
    _on_current_device(x, w, bias, rope_cos, rope_sin, q8, k8, v8, q_scale, k_scale, v_scale, q16, k16, v16)
    _check(load_library().dit_qkv_project_fp8(_ptr(x), _ptr(w), _ptr(bias), _ptr(rope_cos), _ptr(rope_sin), _ptr(q8),
                                              _ptr(k8), _ptr(v8), _ptr(q_scale), _ptr(k_scale), _ptr(v_scale),
                                              _ptr(q16), _ptr(k16), _ptr(v16), B, N, C, H, 128, _stream(stream)),
           "dit_qkv_project_fp8")


def dit_attn_merge(o_parts, lse_parts, out, lse_out=None, dtype: int = DIT_BF16, stream=None) -> None:
    """out (and lse_out) <- merge of R partial results (lists of [B, H, N, D] outputs and [B, H, N] lses)
    over disjoint key sets."""
    import torch
    R = len(o_parts)
    _require(1 <= R <= DIT_MERGE_MAX_PARTS and len(lse_parts) == R, "need 1..16 parts with one lse each")
    B, H, N, D = out.shape
    part_dtype = torch.float32 if dtype & DIT_PART_F32 else torch.bfloat16
    for o, l in zip(o_parts, lse_parts):
        _require(o.is_cuda and o.dtype == part_dtype and o.is_contiguous() and o.shape == out.shape,
                 "part outputs must be contiguous CUDA tensors of out's shape (fp32 with DIT_PART_F32, else bf16)")
        _require(l.is_cuda and l.dtype == torch.float32 and l.is_contiguous() and tuple(l.shape) == (B, H, N),
                 "part lses must be contiguous CUDA fp32 [B, H, N]")
    out_dtype = torch.float32 if dtype & DIT_OUT_F32 else torch.bfloat16
    _require(out.is_cuda and out.dtype == out_dtype and out.is_contiguous(), "out must be contiguous CUDA")
    if lse_out is not None:
        _require(lse_out.is_cuda and lse_out.dtype == torch.float32 and lse_out.is_contiguous() and
                 tuple(lse_out.shape) == (B, H, N), "lse_out must be contiguous CUDA fp32 [B, H, N]")
    _on_current_device(out, lse_out)       # the parts may be a peer GPU's memory, read over NVLink
    optr = (ctypes.c_void_p * R)(*[o.data_ptr() for o in o_parts])
    lptr = (ctypes.c_void_p * R)(*[l.data_ptr() for l in lse_parts])
    _check(load_library().dit_attn_merge(ctypes.cast(optr, ctypes.c_void_p), ctypes.cast(lptr, ctypes.c_void_p), R,
                                         _ptr(out), _ptr(lse_out), B, H, N, D, dtype, _stream(stream)),
           "dit_attn_merge")


def dit_attn_get_status(stream=None) -> int:
    """Synchronise the stream, return and clear the device status word."""
    st = ctypes.c_int(0)
    _check(load_library().dit_attn_get_status(ctypes.byref(st), _stream(stream)), "dit_attn_get_status")
    return st.value


def dit_attn_status_string(status: int) -> str:
    return load_library().dit_attn_status_string(int(status)).decode()


# ----------------------------------------------------------- allocating helpers
def rope_table(pos, axes=(16, 56, 56), theta: float = 10000.0, stream=None):
    """Allocate and fill (cos, sin) tables for CUDA int32 positions [N, 3]."""
    import torch
    N = pos.shape[0]
    c = torch.empty((N, 64), dtype=torch.float32, device=pos.device)
    s = torch.empty_like(c)
    dit_rope_table_build(pos, axes, theta, c, s, stream)
    return c, s


def _flags(out_f32, k_rotated, v_f16, qk_split):
    return ((DIT_OUT_F32 if out_f32 else 0) | (DIT_K_ROTATED if k_rotated else 0) | (DIT_V_F16 if v_f16 else 0) |
            (DIT_QK_SPLIT if qk_split else 0))


def forward(q, k, v, rope_cos=None, rope_sin=None, n_txt: int = 0, out_f32: bool = False, with_lse: bool = True,
            k_rotated: bool = False, v_f16: bool = False, qk_split: bool = False, stream=None):
    """Allocate out (and lse) and run dit_attn_forward; returns (out, lse).  qk_split: k, v are the
    operands of prepare_kv_split (v_f16 is implied)."""
    import torch
    B, H, N, D = q.shape
    out = torch.empty(q.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if with_lse else None
    flags = _flags(out_f32, k_rotated, v_f16 or qk_split, qk_split)
    dit_attn_forward(q, k, v, rope_cos, rope_sin, out, lse, n_txt, N - n_txt, DIT_BF16 | flags, stream)
    return out, lse


def prepare_kv_split(k, v, rope_cos=None, rope_sin=None, stream=None):
    """Allocate and fill (k_split [2, B, H, N, D] fp16, v_f16) for the split form (DIT_QK_SPLIT)."""
    import torch
    k_split = torch.empty((2,) + tuple(k.shape), dtype=torch.float16, device=k.device)
    v_f16 = torch.empty(v.shape, dtype=torch.float16, device=v.device)
    dit_attn_prepare_kv_split(k, v, rope_cos, rope_sin, k_split, v_f16, stream)
    return k_split, v_f16


def forward_kv(q, k, v, q_cos=None, q_sin=None, out_f32: bool = False, with_lse: bool = True,
               k_rotated: bool = False, v_f16: bool = False, qk_split: bool = False, stream=None):
    """Allocate out (and lse) and run dit_attn_forward_kv (queries q against the keys / values k, v);
    returns (out, lse)."""
    import torch
    B, H, N_q, D = q.shape
    out = torch.empty(q.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N_q), dtype=torch.float32, device=q.device) if with_lse else None
    dit_attn_forward_kv(q, k, v, q_cos, q_sin, out, lse, DIT_BF16 | _flags(out_f32, k_rotated, v_f16 or qk_split,
                                                                        qk_split), stream)
    return out, lse


def qkv_project_fp8(x, w, bias=None, rope_cos=None, rope_sin=None, with_bf16: bool = False, stream=None):
    """Allocate and fill the FP8 attention operands from the QKV projection of x [B, N, C] with w [3 H 128, C]:
    returns (q8, k8, v8, q_scale, k_scale, v_scale, q16, k16, v16); the bf16 tensors are None unless with_bf16."""
    import torch
    B, N, _ = x.shape
    H = w.shape[0] // 384
    codes = [torch.empty((B, H, N, 128), dtype=torch.uint8, device=x.device) for _ in range(3)]
    scales = [torch.empty((B, H, (N + 63) // 64), dtype=torch.float32, device=x.device) for _ in range(3)]
    y16 = [torch.empty((B, H, N, 128), dtype=torch.bfloat16, device=x.device) if with_bf16 else None
           for _ in range(3)]
    dit_qkv_project_fp8(x, w, bias, rope_cos, rope_sin, *codes, *scales, *y16, stream=stream)
    return (*codes, *scales, *y16)


def merge(o_parts, lse_parts, out_f32: bool = False, with_lse: bool = True, stream=None):
    """Allocate out (and lse) and run dit_attn_merge; returns (out, lse)."""
    import torch
    o0 = o_parts[0]
    out = torch.empty(o0.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, device=o0.device)
    lse = torch.empty(o0.shape[:3], dtype=torch.float32, device=o0.device) if with_lse else None
    flags = (DIT_PART_F32 if o0.dtype == torch.float32 else 0) | (DIT_OUT_F32 if out_f32 else 0)
    dit_attn_merge(o_parts, lse_parts, out, lse, DIT_BF16 | flags, stream)
    return out, lse


def forward_host(q, k, v, rope_cos=None, rope_sin=None, n_txt: int = 0, out_f32: bool = False,
                 with_lse: bool = True, chunk_heads: int = 4, workspace=None, pin: bool = True, stream=None):
    """Attention of CPU q, k, v through dit_attn_forward_host; allocates (pinned) CPU outputs and, if none is
    given, the device workspace.  Returns (out, lse) once the results are on the host."""
    import torch
    B, H, N, D = q.shape
    out = torch.empty(q.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, pin_memory=pin)
    lse = torch.empty((B, H, N), dtype=torch.float32, pin_memory=pin) if with_lse else None
    dtype = DIT_BF16 | (DIT_OUT_F32 if out_f32 else 0)
    if workspace is None:
        nbytes = dit_attn_forward_host_workspace(B, H, N, dtype, chunk_heads)
        workspace = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    dit_attn_forward_host(q, k, v, rope_cos, rope_sin, out, lse, n_txt, N - n_txt, workspace, dtype, chunk_heads,
                          stream)
    s = stream if stream is not None else torch.cuda.current_stream()
    s.synchronize()
    return out, lse


def forward_sparse(q, k, v, kv_mask, rope_cos=None, rope_sin=None, n_txt: int = 0, out_f32: bool = False,
                   with_lse: bool = True, k_rotated: bool = False, v_f16: bool = False, stream=None):
    """Allocate out (and lse) and run dit_attn_forward_sparse; returns (out, lse)."""
    import torch
    B, H, N, D = q.shape
    out = torch.empty(q.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if with_lse else None
    flags = (DIT_OUT_F32 if out_f32 else 0) | (DIT_K_ROTATED if k_rotated else 0) | (DIT_V_F16 if v_f16 else 0)
    dit_attn_forward_sparse(q, k, v, rope_cos, rope_sin, kv_mask, out, lse, n_txt, N - n_txt, DIT_BF16 | flags,
                            stream)
    return out, lse


def forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, n_txt: int = 0, out_f32: bool = False,
                with_lse: bool = True, stream=None):
    """Allocate out (and lse) and run dit_attn_forward_fp8; returns (out, lse)."""
    import torch
    B, H, N, D = q8.shape
    out = torch.empty(q8.shape, dtype=torch.float32 if out_f32 else torch.bfloat16, device=q8.device)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=q8.device) if with_lse else None
    dit_attn_forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, out, lse, n_txt, N - n_txt,
                         DIT_FP8_E4M3 | (DIT_OUT_F32 if out_f32 else 0), stream)
    return out, lse
