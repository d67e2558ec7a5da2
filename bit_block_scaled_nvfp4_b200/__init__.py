"""QK4V8 block-scaled low-bit FlashAttention for B200 (sm_100a).

The product is the C-ABI library ``libqk4v8.so`` (include/qk4v8.h); ``api`` is its thin torch
binding, ``workloads`` the seeded synthetic inputs, ``build`` the in-tree nvcc build.
"""
from .api import (  # noqa: F401
    MXFP8V, NVFP4Tensor, PagedKV, attn_qk4v8_decode_paged, attn_qk4v8_fwd, check_status,
    qk4v8_attention, quantize_mxfp8_v, quantize_nvfp4, tile_score_select,
)
