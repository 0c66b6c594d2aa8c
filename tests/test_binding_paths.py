"""Every wrapper of the Python binding, run end to end on a machine without a
GPU: its checks pass, its arguments match the C signature, the C entry point
accepts them and fails at its first CUDA call, and the binding turns that
status into DitError.  The CUDA tensors are stand-ins carrying the metadata the
binding reads and an aligned address the library never dereferences here.
Skipped where a GPU is present: there such addresses could reach a kernel."""
import pytest
import torch

import diffusion_transformer_joint_attn_b200 as dit

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="stand-in addresses must never reach a real GPU")


class OnGpu:
    """A CUDA tensor's metadata and a 16-byte aligned address, no storage."""
    _next = 1 << 24

    def __init__(self, shape, dtype):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.is_cuda = True
        self.device = torch.device("cuda", 0)
        OnGpu._next += 1 << 24
        self._addr = OnGpu._next

    def dim(self):
        return len(self.shape)

    def is_contiguous(self):
        return True

    def data_ptr(self):
        return self._addr

    def numel(self):
        return self.shape.numel()

    def element_size(self):
        return torch.empty((), dtype=self.dtype).element_size()


@pytest.fixture(autouse=True)
def current_device_zero(monkeypatch):
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)


B, H, NT, NI, D = 1, 2, 8, 24, 128
N = NT + NI
bf16, f16, f32, u8, i32 = torch.bfloat16, torch.float16, torch.float32, torch.uint8, torch.int32


def fails_at_cuda(fn):
    with pytest.raises(dit.DitError) as e:
        fn()
    assert e.value.status == dit.DIT_ERR_CUDA


def test_rotary_wrappers():
    c, s = OnGpu((N, 64), f32), OnGpu((N, 64), f32)
    fails_at_cuda(lambda: dit.dit_rope_table_build(OnGpu((N, 3), i32), (16, 56, 56), 1e4, c, s, stream=0))
    x = OnGpu((B, H, N, D), bf16)
    fails_at_cuda(lambda: dit.dit_rope_apply(x, c, s, OnGpu((B, H, N, D), bf16), stream=0))
    fails_at_cuda(lambda: dit.dit_attn_prepare_kv(x, x, c, s, OnGpu((B, H, N, D), bf16), OnGpu((B, H, N, D), f16),
                                                  stream=0))


def test_forward_wrappers():
    q = OnGpu((B, H, N, D), bf16)
    c, s = OnGpu((N, 64), f32), OnGpu((N, 64), f32)
    out, lse = OnGpu((B, H, N, D), f32), OnGpu((B, H, N), f32)
    fails_at_cuda(lambda: dit.dit_attn_forward(q, q, q, c, s, out, lse, NT, NI, dit.DIT_OUT_F32, stream=0))
    fails_at_cuda(lambda: dit.dit_attn_forward(q, q, OnGpu((B, H, N, D), f16), c, s, OnGpu((B, H, N, D), bf16), None,
                                               NT, NI, dit.DIT_K_ROTATED | dit.DIT_V_F16, stream=0))
    mask = OnGpu((B, H, 1, 1), u8)
    fails_at_cuda(lambda: dit.dit_attn_forward_sparse(q, q, q, c, s, mask, out, lse, NT, NI, dit.DIT_OUT_F32,
                                                      stream=0))


def test_split_and_key_set_wrappers():
    q = OnGpu((B, H, N, D), bf16)
    c, s = OnGpu((N, 64), f32), OnGpu((N, 64), f32)
    k_split, v16 = OnGpu((2, B, H, N, D), f16), OnGpu((B, H, N, D), f16)
    fails_at_cuda(lambda: dit.dit_attn_prepare_kv_split(q, q, c, s, k_split, v16, stream=0))
    fails_at_cuda(lambda: dit.dit_attn_prepare_kv_split(q, q, None, None, k_split, v16, stream=0))
    out, lse = OnGpu((B, H, N, D), f32), OnGpu((B, H, N), f32)
    fails_at_cuda(lambda: dit.dit_attn_forward(q, k_split, v16, c, s, out, lse, NT, NI,
                                               dit.DIT_QK_SPLIT | dit.DIT_V_F16 | dit.DIT_OUT_F32, stream=0))
    with pytest.raises(ValueError, match="DIT_QK_SPLIT"):    # a bf16 k is not the split operand
        dit.dit_attn_forward(q, q, v16, c, s, out, lse, NT, NI, dit.DIT_QK_SPLIT | dit.DIT_V_F16 | dit.DIT_OUT_F32,
                             stream=0)
    # queries of tokens 0..N-1 against a shard of 40 keys
    Nkv = 40
    kr, vk = OnGpu((B, H, Nkv, D), bf16), OnGpu((B, H, Nkv, D), f16)
    fails_at_cuda(lambda: dit.dit_attn_forward_kv(q, kr, vk, c, s, out, lse,
                                                  dit.DIT_K_ROTATED | dit.DIT_V_F16 | dit.DIT_OUT_F32, stream=0))
    ks = OnGpu((2, B, H, Nkv, D), f16)
    fails_at_cuda(lambda: dit.dit_attn_forward_kv(q, ks, vk, c, s, out, None,
                                                  dit.DIT_QK_SPLIT | dit.DIT_V_F16 | dit.DIT_OUT_F32, stream=0))
    with pytest.raises(ValueError, match="N_kv"):
        dit.dit_attn_forward_kv(q, OnGpu((B, H, Nkv + 1, D), bf16), vk, c, s, out, lse,
                                dit.DIT_K_ROTATED | dit.DIT_V_F16 | dit.DIT_OUT_F32, stream=0)
    with pytest.raises(ValueError, match="rope tables"):     # the query tables have N_q rows
        dit.dit_attn_forward_kv(q, kr, vk, OnGpu((Nkv, 64), f32), OnGpu((Nkv, 64), f32), out, lse,
                                dit.DIT_K_ROTATED | dit.DIT_V_F16 | dit.DIT_OUT_F32, stream=0)


def test_projection_wrapper():
    C, H = 256, 2
    x, w = OnGpu((B, N, C), bf16), OnGpu((3 * H * 128, C), bf16)
    codes = [OnGpu((B, H, N, D), u8) for _ in range(3)]
    scales = [OnGpu((B, H, (N + 63) // 64), f32) for _ in range(3)]
    y16 = [OnGpu((B, H, N, D), bf16) for _ in range(3)]
    c, s = OnGpu((N, 64), f32), OnGpu((N, 64), f32)
    fails_at_cuda(lambda: dit.dit_qkv_project_fp8(x, w, OnGpu((3 * H * 128,), f32), c, s, *codes, *scales, *y16,
                                                  stream=0))
    fails_at_cuda(lambda: dit.dit_qkv_project_fp8(x, w, None, None, None, *codes, *scales, stream=0))
    with pytest.raises(ValueError, match="scales"):
        dit.dit_qkv_project_fp8(x, w, None, None, None, *codes, scales[0], scales[1], OnGpu((B, H, 2), f32),
                                stream=0)


def test_fp8_wrappers():
    x = OnGpu((B, H, N, D), bf16)
    codes, scale = OnGpu((B, H, N, D), u8), OnGpu((B, H, 1), f32)
    fails_at_cuda(lambda: dit.dit_attn_quantize_fp8(x, OnGpu((N, 64), f32), OnGpu((N, 64), f32), codes, scale,
                                                    stream=0))
    fails_at_cuda(lambda: dit.dit_attn_quantize_fp8(x, None, None, codes, scale, stream=0))
    fails_at_cuda(lambda: dit.dit_attn_forward_fp8(codes, codes, codes, scale, scale, scale,
                                                   OnGpu((B, H, N, D), bf16), OnGpu((B, H, N), f32), NT, NI,
                                                   stream=0))


def test_merge_wrapper():
    parts = [OnGpu((B, H, N, D), bf16) for _ in range(3)]
    lses = [OnGpu((B, H, N), f32) for _ in range(3)]
    fails_at_cuda(lambda: dit.dit_attn_merge(parts, lses, OnGpu((B, H, N, D), f32), OnGpu((B, H, N), f32),
                                             dit.DIT_OUT_F32, stream=0))


def test_host_buffer_wrapper():
    q = torch.zeros(B, H, N, D, dtype=bf16)
    out, lse = torch.zeros(B, H, N, D, dtype=bf16), torch.zeros(B, H, N, dtype=f32)
    nbytes = dit.dit_attn_forward_host_workspace(B, H, N, dit.DIT_BF16, 4)
    assert nbytes > 0
    ws = OnGpu((nbytes,), u8)
    fails_at_cuda(lambda: dit.dit_attn_forward_host(q, q, q, OnGpu((N, 64), f32), OnGpu((N, 64), f32), out, lse,
                                                    NT, NI, ws, dit.DIT_BF16, 4, stream=0))


def test_a_tensor_on_another_device_is_refused_before_the_library():
    q = OnGpu((B, H, N, D), bf16)
    other = OnGpu((B, H, N, D), bf16)
    other.device = torch.device("cuda", 1)
    with pytest.raises(ValueError, match="one device"):
        dit.dit_attn_forward(q, other, q, None, None, OnGpu((B, H, N, D), bf16), None, NT, NI, stream=0)
