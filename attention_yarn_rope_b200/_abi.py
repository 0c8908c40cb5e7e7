"""ctypes declarations of libgptoss_attn's C ABI (include/gptoss.h).

Argument marshalling only.  The library must exist in-tree (built by
``attention_yarn_rope_b200.build_lib``); a missing library raises, there is
no fallback.
"""

from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptoss_attn.so")
# the same library built with in-kernel range checks (GPTOSS_DEBUG_CHECKS)
DEBUG_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptoss_attn_debug.so")

GPTOSS_OK = 0
GPTOSS_ERR_INVALID_ARG = 1
GPTOSS_ERR_UNSUPPORTED = 2
GPTOSS_ERR_CUDA = 3
GPTOSS_ERR_TIMEOUT = 4

STATUS_NAMES = {
    0: "GPTOSS_OK",
    1: "GPTOSS_ERR_INVALID_ARG",
    2: "GPTOSS_ERR_UNSUPPORTED",
    3: "GPTOSS_ERR_CUDA",
    4: "GPTOSS_ERR_TIMEOUT",
}

# Every symbol include/gptoss.h declares.
EXPORTED = (
    "gptoss_status_string",
    "gptoss_rope_qk",
    "gptoss_attn_fwd",
    "gptoss_attn_fwd_workspace_size",
    "gptoss_attn_fwd_block",
    "gptoss_attn_fwd_block_workspace_size",
    "gptoss_attn_merge",
    "gptoss_qkv_rope_workspace_size",
    "gptoss_qkv_rope",
    "gptoss_attn_decode_workspace_size",
    "gptoss_attn_decode",
    "gptoss_attn_decode_noalloc",
    "gptoss_attn_decode_paged",
    "gptoss_kv_append_paged",
    "gptoss_attn_bwd_workspace_size",
    "gptoss_attn_bwd",
    "gptoss_read_device_status",
    "gptoss_set_wait_limit",
    "gptoss_selftest_wait_timeout",
)


class RopeParams(ctypes.Structure):
    _fields_ = [
        ("base", ctypes.c_double),
        ("factor", ctypes.c_double),
        ("initial_context", ctypes.c_int32),
        ("rotary_dim", ctypes.c_int32),
        ("ntk_alpha", ctypes.c_double),
        ("ntk_beta", ctypes.c_double),
    ]


class Strides(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("tok", ctypes.c_int64), ("head", ctypes.c_int64)]


_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_u32 = ctypes.c_uint32
_f32 = ctypes.c_float
_st = ctypes.c_int  # gptoss_status (enum)

_SIGNATURES = {
    "gptoss_status_string": (ctypes.c_char_p, [_st]),
    "gptoss_rope_qk": (_st, [_vp, Strides, _vp, Strides, _vp, Strides, _vp, Strides, _vp, _vp, _i32, _i32, _i32,
                             _i32, _i32, ctypes.POINTER(RopeParams), _vp]),
    "gptoss_attn_fwd": (_st, [_vp, Strides, _vp, Strides, _vp, Strides, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                              _i32, _i32, _i32, _f32, ctypes.POINTER(RopeParams), _vp, Strides, _vp, _vp,
                              ctypes.c_size_t, _vp]),
    "gptoss_attn_fwd_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32]),
    "gptoss_attn_fwd_block": (_st, [_vp, Strides, _vp, Strides, _vp, Strides, _i32, _i32, _i32, _i32, _i32, _i32,
                                    _i32, _i32, _f32, ctypes.POINTER(RopeParams), _vp, _vp, _vp, ctypes.c_size_t,
                                    _vp]),
    "gptoss_attn_fwd_block_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32, _i32]),
    "gptoss_attn_merge": (_st, [_vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _vp, Strides, _vp, _vp]),
    "gptoss_qkv_rope_workspace_size": (ctypes.c_size_t, [_i32, _i32]),
    "gptoss_qkv_rope": (_st, [_vp, ctypes.c_int64, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32,
                              ctypes.POINTER(RopeParams), _vp, Strides, _vp, Strides, _vp, Strides, _vp,
                              ctypes.c_size_t, _vp]),
    "gptoss_attn_decode_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32, _i32]),
    "gptoss_attn_decode": (_st, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                 ctypes.POINTER(RopeParams), _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "gptoss_attn_decode_noalloc": (_st, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                         ctypes.POINTER(RopeParams), _vp, _vp, _vp]),
    "gptoss_attn_decode_paged": (_st, [_vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32,
                                       _i32, _i32, _f32, ctypes.POINTER(RopeParams), _vp, _vp, _vp,
                                       ctypes.c_size_t, _vp]),
    "gptoss_kv_append_paged": (_st, [_vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                     ctypes.POINTER(RopeParams), _vp]),
    "gptoss_attn_bwd_workspace_size": (ctypes.c_size_t, [_i32, _i32, _i32, _i32]),
    "gptoss_attn_bwd": (_st, [_vp, Strides, _vp, Strides, _vp, Strides, _vp, Strides, _vp, Strides, _vp, _vp, _vp,
                              _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, ctypes.POINTER(RopeParams), _vp,
                              _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "gptoss_read_device_status": (_st, [ctypes.POINTER(_i32), _i32, _vp]),
    "gptoss_set_wait_limit": (_st, [_u32]),
    "gptoss_selftest_wait_timeout": (_st, [_u32, _vp, _vp]),
}

_lib = None


def _open(path: str) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(
            f"{os.path.basename(path)} not found at {path}; build it with "
            "`python -m attention_yarn_rope_b200.build_lib` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load() -> ctypes.CDLL:
    """Load the in-tree library once.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        _lib = _open(LIB_PATH)
    return _lib


def load_debug() -> ctypes.CDLL:
    """The range-checking build (``build_lib --debug-checks``), loaded on its own."""
    return _open(DEBUG_LIB_PATH)


class GptossError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


def check(fn: str, status: int) -> None:
    if status != GPTOSS_OK:
        raise GptossError(fn, status)
