"""The allocation-free decode entry point (attn_qk4v8_decode_paged_noalloc).

Some callers cannot give the library device memory for scratch: an engine that fixed all its
buffers at start-up and forbids allocation in its step loop, a plugin inside a framework that
owns all device memory, or a host program that links only this library. For them the library
keeps the decode's split partials in its own fixed device buffer. These tests call that entry
point through the C ABI and compare it with the workspace-taking entry point, twice in a row
(the second call reuses the buffer the first one left behind), and check that a request too
big for the buffer is refused before anything is launched. The file sorts last so that a run
stopping at the first failure has run every other test first.
"""
import ctypes as C
import math

import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import _lib, api, paged
from helpers import assert_attention_close, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _small_cache():
    g = torch.Generator().manual_seed(21)
    lens = [700, 129, 2000]
    hkv, hq, d = 2, 8, 128
    pages_per = [(n + 63) // 64 for n in lens]
    perm = torch.randperm(sum(pages_per), generator=g)
    table = torch.full((len(lens), max(pages_per)), -1, dtype=torch.int32)
    cache = paged.empty_cache(sum(pages_per), hkv, d, 0.0625, DEV)
    off = 0
    for s, n in enumerate(lens):
        table[s, :pages_per[s]] = perm[off:off + pages_per[s]].int()
        off += pages_per[s]
        k = (torch.randn(n, hkv, d, generator=g) * 3).to(torch.bfloat16)
        v = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
        paged.write_sequence(cache, k.to(DEV), v.to(DEV), table[s, :pages_per[s]])
    q = torch.randn(len(lens), hq, d, generator=g).to(torch.bfloat16)
    return cache, table.to(DEV), torch.tensor(lens, dtype=torch.int32, device=DEV), q, max(lens)


def test_noalloc_decode_matches_workspace_entry_point_twice():
    cache, table, ctx, q, max_ctx = _small_cache()
    q4 = api.quantize_nvfp4(q.to(DEV))
    want = api.attn_qk4v8_decode_paged(q4, cache, table, ctx, max_ctx, 256,
                                       out_dtype=torch.float32)
    for _ in range(2):
        got = api.attn_qk4v8_decode_paged_noalloc(q4, cache, table, ctx, max_ctx, 256,
                                                  out_dtype=torch.float32)
        assert api.check_status() == 0
        assert_attention_close(f32(got), f32(want).astype(np.float64), "no-alloc decode")
        assert torch.equal(got, want)                  # same kernels, deterministic


def test_noalloc_decode_refuses_requests_beyond_its_buffer():
    cache, table, ctx, q, _ = _small_cache()
    q4 = api.quantize_nvfp4(q.to(DEV))
    out = torch.empty(3, 8, 128, dtype=torch.float32, device=DEV)
    # 3 sequences x 8 heads x splits x 130 floats: a one-split-per-128-keys request over a
    # context bound of 2^20 keys needs 3 * 8 * 8192 * 520 bytes > 16 MiB
    p = api.decode_params(q4, cache, table, ctx, 1 << 20, 128, out)
    lib = _lib.load()
    assert lib.attn_qk4v8_decode_workspace_size(C.byref(p)) > _lib.NOALLOC_DECODE_SCRATCH_BYTES
    st = lib.attn_qk4v8_decode_paged_noalloc(C.byref(p), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == _lib.QK4V8_ERR_UNSUPPORTED
    assert api.check_status() == 0
