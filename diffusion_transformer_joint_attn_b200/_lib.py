"""Loader of the in-tree shared library libdit_attn.so (ctypes)."""
from __future__ import annotations

import ctypes
import os
import threading

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB = None
_LOCK = threading.Lock()

_VP = ctypes.c_void_p
_I = ctypes.c_int

# name -> (restype, argtypes), mirroring include/dit_attn.h
SIGNATURES = {
    "dit_rope_table_build": (_I, [_VP, _I, _I, ctypes.POINTER(ctypes.c_int32), ctypes.c_double, _VP, _VP, _VP]),
    "dit_rope_apply": (_I, [_VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "dit_attn_prepare_kv": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "dit_attn_prepare_kv_split": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "dit_attn_forward": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP]),
    "dit_attn_forward_kv": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP]),
    "dit_attn_forward_host_workspace": (ctypes.c_size_t, [_I, _I, _I, _I, _I, _I]),
    "dit_attn_forward_host": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP, ctypes.c_size_t,
                                   _I, _VP]),
    "dit_attn_forward_host_static": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _I, _VP]),
    "dit_attn_forward_sparse": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP]),
    "dit_attn_quantize_fp8": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _VP]),
    "dit_attn_forward_fp8": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _VP]),
    "dit_qkv_project_fp8": (_I, [_VP] * 14 + [_I, _I, _I, _I, _I, _VP]),
    "dit_attn_merge": (_I, [_VP, _VP, _I, _VP, _VP, _I, _I, _I, _I, _I, _VP]),
    "dit_attn_wait_selftest": (_I, [ctypes.c_longlong, _VP]),
    "dit_attn_get_status": (_I, [ctypes.POINTER(ctypes.c_int), _VP]),
    "dit_attn_status_string": (ctypes.c_char_p, [_I]),
    "dit_attn_last_cuda_error": (_I, []),
    "dit_attn_last_cuda_error_string": (ctypes.c_char_p, []),
}


def library_path() -> str:
    return os.path.join(_PKG_DIR, "libdit_attn.so")


def load_library():
    """The loaded library; raises if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    with _LOCK:
        if _LIB is None:
            path = library_path()
            if not os.path.exists(path):
                raise RuntimeError("libdit_attn.so is not built (python -m diffusion_transformer_joint_attn_b200.build)")
            lib = ctypes.CDLL(path)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _LIB = lib
    return _LIB
