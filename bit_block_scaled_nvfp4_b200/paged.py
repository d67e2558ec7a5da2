"""Fill a paged NVFP4-K / MXFP8-V KV cache from dense per-sequence K/V.

Quantization runs in the library's kernels (quantize_nvfp4 with the cache's fixed tensor
scale, quantize_mxfp8_v); torch only moves the resulting bytes into 64-token pages at the
physical ids of the page table. This is cache set-up, outside the decode step.
"""
from __future__ import annotations

import torch

from .api import PagedKV, quantize_mxfp8_v, quantize_nvfp4

PAGE = 64


def empty_cache(num_pages: int, kv_heads: int, head_dim: int, k_tensor_scale: float,
                device) -> PagedKV:
    d = head_dim
    return PagedKV(
        k_pages=torch.zeros(num_pages, kv_heads, PAGE, d // 2, dtype=torch.uint8, device=device),
        k_scales=torch.zeros(num_pages, kv_heads, PAGE, d // 16, dtype=torch.uint8, device=device),
        k_tensor_scale=torch.tensor([k_tensor_scale], dtype=torch.float32, device=device),
        v_pages=torch.zeros(num_pages, kv_heads, d, PAGE, dtype=torch.uint8, device=device),
        v_scales=torch.full((num_pages, kv_heads, d, 2), 127, dtype=torch.uint8, device=device),
    )


def empty_tail(num_seqs: int, kv_heads: int, head_dim: int, dtype, device) -> torch.Tensor:
    """The per-sequence incomplete-V-group state that kv_append_paged reads and updates."""
    return torch.zeros(num_seqs, kv_heads, head_dim, 32, dtype=dtype, device=device)


def write_sequence(cache: PagedKV, k: torch.Tensor, v: torch.Tensor, pages: torch.Tensor) -> None:
    """Quantize one sequence's K, V ([len, Hkv, D] on the cache's device) into the physical
    pages ``pages`` (int tensor of ceil(len/64) ids)."""
    n, hkv, d = k.shape
    n_pages = (n + PAGE - 1) // PAGE
    npad = n_pages * PAGE
    kh = torch.zeros(hkv, npad, d, dtype=k.dtype, device=k.device)
    kh[:, :n] = k.transpose(0, 1)
    k4 = quantize_nvfp4(kh, tensor_scale=float(cache.k_tensor_scale.item()))
    pages = pages.to(device=k.device, dtype=torch.long)
    cache.k_pages[pages] = k4.codes.view(hkv, n_pages, PAGE, d // 2).transpose(0, 1)
    cache.k_scales[pages] = k4.scales.view(hkv, n_pages, PAGE, d // 16).transpose(0, 1)
    v8 = quantize_mxfp8_v(v.transpose(0, 1).contiguous())          # codes [Hkv, D, n_pad128]
    vc = v8.codes[:, :, :npad].reshape(hkv, d, n_pages, PAGE).permute(2, 0, 1, 3)
    vs = v8.scales[:, :, :npad // 32].reshape(hkv, d, n_pages, 2).permute(2, 0, 1, 3)
    cache.v_pages[pages] = vc
    cache.v_scales[pages] = vs
