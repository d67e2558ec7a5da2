"""ctypes view of libqk4v8.so: signatures and parameter structs of include/qk4v8.h.

Nothing here computes; it only loads the library and describes its ABI. The library must be
built in-tree (``python -m bit_block_scaled_nvfp4_b200.build``); loading fails loudly if it is
missing. There is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libqk4v8.so")

QK4V8_OK = 0
QK4V8_ERR_INVALID_ARG = 1
QK4V8_ERR_UNSUPPORTED = 2
QK4V8_ERR_CUDA = 3
QK4V8_ERR_TIMEOUT = 4
QK4V8_ERR_BOUNDS = 5
QK4V8_F16 = 0
QK4V8_BF16 = 1
QK4V8_F32 = 2
#: Size of the library's fixed scratch buffer behind attn_qk4v8_decode_paged_noalloc.
NOALLOC_DECODE_SCRATCH_BYTES = 16 * 1024 * 1024

vp = C.c_void_p
i32 = C.c_int32
i64 = C.c_int64
f32 = C.c_float
sz = C.c_size_t


class FwdParams(C.Structure):
    _fields_ = [
        ("q_codes", vp), ("q_scales", vp), ("q_tensor_scale", vp),
        ("k_codes", vp), ("k_scales", vp), ("k_tensor_scale", vp),
        ("v_codes", vp), ("v_scales", vp),
        ("batch", i32), ("q_heads", i32), ("kv_heads", i32), ("n_q", i32), ("n_k", i32),
        ("head_dim", i32), ("causal", i32), ("softmax_scale", f32),
        ("fp16_bitmap", vp), ("q16", vp), ("k16", vp), ("v16", vp),
        ("out_dtype", i32), ("out", vp), ("lse", vp), ("p_underflow_aware", i32),
        ("q2_codes", vp), ("q2_scales", vp), ("qk16_dtype", i32),
    ]


class DecodeParams(C.Structure):
    _fields_ = [
        ("q_codes", vp), ("q_scales", vp), ("q_tensor_scale", vp),
        ("k_pages", vp), ("k_page_scales", vp), ("k_tensor_scale", vp),
        ("v_pages", vp), ("v_page_scales", vp),
        ("page_table", vp), ("context_lens", vp),
        ("num_seqs", i32), ("num_pages", i32), ("max_pages", i32), ("q_heads", i32),
        ("kv_heads", i32), ("head_dim", i32), ("max_context", i32), ("split_tokens", i32),
        ("softmax_scale", f32), ("out_dtype", i32), ("out", vp), ("lse", vp),
        ("p_underflow_aware", i32), ("q2_codes", vp), ("q2_scales", vp),
    ]


class AppendParams(C.Structure):
    _fields_ = [
        ("k_new", vp), ("v_new", vp), ("dtype", i32),
        ("cu_new", vp), ("lens", vp), ("page_table", vp),
        ("k_pages", vp), ("k_page_scales", vp), ("k_tensor_scale", vp),
        ("v_pages", vp), ("v_page_scales", vp), ("v_tail", vp),
        ("num_seqs", i32), ("num_pages", i32), ("max_pages", i32), ("kv_heads", i32),
        ("head_dim", i32), ("max_new", i32),
    ]


class QkvParams(C.Structure):
    _fields_ = [
        ("q", vp), ("k", vp), ("v", vp), ("dtype", i32), ("head_dim", i32),
        ("q_rows", i64), ("k_rows", i64), ("v_bh", i32), ("v_tokens", i32),
        ("q_codes", vp), ("q_scales", vp), ("q_tensor_scale", vp),
        ("k_codes", vp), ("k_scales", vp), ("k_tensor_scale", vp),
        ("v_codes", vp), ("v_scales", vp),
        ("q16", vp), ("k16", vp), ("v16", vp),
    ]


#: name -> (restype, argtypes); exactly the functions include/qk4v8.h declares.
SIGNATURES = {
    "qk4v8_version": (C.c_int, []),
    "qk4v8_status_string": (C.c_char_p, [i32]),
    "qk4v8_check_status": (i32, [vp]),
    "qk4v8_struct_size": (sz, [i32]),
    "qk4v8_timeout_site": (C.c_uint64, []),
    "qk4v8_selftest_wait_timeout": (i32, [vp]),
    "qk4v8_selftest_device_once": (i32, [i32]),
    "quantize_nvfp4_workspace_size": (sz, []),
    "quantize_nvfp4": (i32, [vp, i32, i64, i32, i64, f32, vp, vp, vp, vp, vp, sz, vp]),
    "quantize_mxfp8_v": (i32, [vp, i32, i32, i32, i32, vp, vp, vp, vp]),
    "quantize_qkv_workspace_size": (sz, []),
    "quantize_qkv": (i32, [C.POINTER(QkvParams), vp, sz, vp]),
    "quantize_nvfp4_residual": (i32, [vp, i32, i64, i32, i64, vp, vp, vp, vp, vp, vp]),
    "quantize_nvfp4_searched": (i32, [vp, i32, i64, i32, i64, f32, vp, vp, vp, vp, vp, sz, vp]),
    "qk_smooth_rotate": (i32, [vp, i32, i64, i32, vp, i32, vp, vp]),
    "tile_score_select_workspace_size": (sz, [i32, i32, i32, i32]),
    "tile_score_select": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                vp, vp, vp, vp, sz, vp]),
    "attn_qk4v8_fwd": (i32, [C.POINTER(FwdParams), vp]),
    "attn_qk4v8_decode_workspace_size": (sz, [C.POINTER(DecodeParams)]),
    "attn_qk4v8_decode_paged": (i32, [C.POINTER(DecodeParams), vp, sz, vp]),
    "attn_qk4v8_decode_paged_noalloc": (i32, [C.POINTER(DecodeParams), vp]),
    "kv_append_paged": (i32, [C.POINTER(AppendParams), vp]),
}

_LIB = None


class QK4V8Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def load():
    """Load libqk4v8.so (once). Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m bit_block_scaled_nvfp4_b200.build`")
        lib = C.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def status_string(status: int) -> str:
    return load().qk4v8_status_string(status).decode()


def check(status: int, where: str) -> None:
    if status != QK4V8_OK:
        raise QK4V8Error(status, where)
