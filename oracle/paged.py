"""Oracle — paged KV-cache layout (TEST INFRASTRUCTURE ONLY; see oracle/formats.py).

The decode path of the sns.style BitDecoding-FP4 summary reads a paged KV cache once per
step (system section: stacked-query MMA on a paged KV cache); the hotelren.com MpFA article
§6 combines QK4V8 with paged KV management. Page size 64 tokens. Per page and KV head:

    K codes  [64, d/2]   NVFP4 E2M1 pairs, one row per token      (cache-wide FP32 scale)
    K scales [64, d/16]  E4M3
    V codes  [d, 64]     E4M3, token-contiguous per channel
    V scales [d, 2]      E8M0, one per 32 tokens

A sequence's logical page p lives at physical page page_table[seq, p]. This module only
moves bytes between the dense per-sequence form and the page form; the quantization itself
is ``oracle.quant``.
"""
from __future__ import annotations

import numpy as np

from .quant import mxfp8_quantize_v, nvfp4_quantize

PAGE = 64


def quantize_sequence(k: np.ndarray, v: np.ndarray, k_tensor_scale: float):
    """k, v: [len, Hkv, d] float values of one sequence. Returns dense-per-head codes:
    kc [Hkv, len, d/2], ks [Hkv, len, d/16], vc [Hkv, d, len_pad128], vs [Hkv, d, len_pad128/32].
    """
    kh = np.swapaxes(np.asarray(k, dtype=np.float32), 0, 1)       # [Hkv, len, d]
    vh = np.swapaxes(np.asarray(v, dtype=np.float32), 0, 1)
    kc, ks, _ = nvfp4_quantize(kh, tensor_scale=k_tensor_scale)
    vc, vs = mxfp8_quantize_v(vh)
    return kc, ks, vc, vs


def sequence_pages(kc, ks, vc, vs, length: int):
    """Cut one sequence's dense codes into its logical pages, padding the last page.

    Returns arrays [n_pages, Hkv, ...] in the page layout above.
    """
    hkv, _, dh = kc.shape
    d = vc.shape[1]
    n_pages = (length + PAGE - 1) // PAGE
    kcp = np.zeros((n_pages, hkv, PAGE, dh), dtype=np.uint8)
    ksp = np.zeros((n_pages, hkv, PAGE, ks.shape[2]), dtype=np.uint8)
    vcp = np.zeros((n_pages, hkv, d, PAGE), dtype=np.uint8)
    vsp = np.zeros((n_pages, hkv, d, PAGE // 32), dtype=np.uint8)
    for p in range(n_pages):
        t0, t1 = p * PAGE, min((p + 1) * PAGE, length)
        kcp[p, :, :t1 - t0] = kc[:, t0:t1]
        ksp[p, :, :t1 - t0] = ks[:, t0:t1]
        vcp[p] = vc[:, :, t0:t0 + PAGE]
        vsp[p] = vs[:, :, t0 // 32:t0 // 32 + PAGE // 32]
    return kcp, ksp, vcp, vsp


def gather_sequence(k_pages, k_scales, v_pages, v_scales, table_row, length: int):
    """Read one sequence back from physical pages into dense per-head codes
    (the inverse of ``sequence_pages`` followed by placement at ``table_row``)."""
    n_pages = (length + PAGE - 1) // PAGE
    ids = np.asarray(table_row[:n_pages], dtype=np.int64)
    kc = np.concatenate([k_pages[i] for i in ids], axis=1)[:, :length]
    ks = np.concatenate([k_scales[i] for i in ids], axis=1)[:, :length]
    vc = np.concatenate([v_pages[i] for i in ids], axis=2)
    vs = np.concatenate([v_scales[i] for i in ids], axis=2)
    return kc, ks, vc, vs
