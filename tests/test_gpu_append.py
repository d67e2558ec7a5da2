"""GPU parity of quantize-on-append (kv_append_paged) against the oracle: after every append,
each sequence's pages hold exactly the oracle's encoding of its whole prefix (NVFP4 K with the
cache's fixed tensor scale, MXFP8 V per 32-token group), for appends of one token, of chunks
that cross V groups and pages, and of whole prompts; the decode step then reads the same bytes
as from a cache written in one piece."""
import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, paged
from oracle import paged as OP
from helpers import f32

pytestmark = pytest.mark.gpu
DEV = "cuda"
KTS = 2.0 ** -6 * 1.37


def _pages_equal(cache, table_row, k, v, length):
    kc, ks, vc, vs = OP.quantize_sequence(f32(k[:length]), f32(v[:length]), np.float32(KTS))
    want = OP.sequence_pages(kc, ks, vc, vs, length)
    ids = table_row[:(length + 63) // 64].long()
    got = [cache.k_pages[ids], cache.k_scales[ids], cache.v_pages[ids], cache.v_scales[ids]]
    for name, g, w in zip(("K codes", "K scales", "V codes", "V scales"), got, want):
        g = g.cpu().numpy()
        assert np.array_equal(g, w), f"{name} differ at {np.argwhere(g != w)[:4]} (len {length})"


def _run(dtype, lens_total, chunk_plan, hkv=2, seed=0):
    """Append each sequence's tokens in the chunk sizes of chunk_plan (a list of per-call lists
    of new-token counts), checking the pages after every call."""
    d = 128
    S = len(lens_total)
    g = torch.Generator().manual_seed(seed)
    seqs = []
    for n in lens_total:
        k = (torch.randn(n, hkv, d, generator=g) + torch.randn(1, hkv, d, generator=g) * 0.5)
        v = torch.randn(n, hkv, d, generator=g) * torch.exp(torch.randn(n, 1, 1, generator=g))
        seqs.append((k.to(dtype), v.to(dtype)))
    max_pages = max((n + 63) // 64 for n in lens_total)
    num_pages = S * max_pages + 3
    perm = torch.randperm(num_pages, generator=g)[:S * max_pages].view(S, max_pages).to(torch.int32)
    cache = paged.empty_cache(num_pages, hkv, d, KTS, DEV)
    tail = paged.empty_tail(S, hkv, d, dtype, DEV)
    table = perm.to(DEV)
    lens = [0] * S
    for call in chunk_plan:
        ks, vs, cu = [], [], [0]
        for s, n_new in enumerate(call):
            n_new = min(n_new, lens_total[s] - lens[s])
            ks.append(seqs[s][0][lens[s]:lens[s] + n_new])
            vs.append(seqs[s][1][lens[s]:lens[s] + n_new])
            cu.append(cu[-1] + n_new)
        k_new = torch.cat(ks).to(DEV).contiguous()
        v_new = torch.cat(vs).to(DEV).contiguous()
        if k_new.shape[0] == 0:
            continue
        api.kv_append_paged(cache, k_new, v_new, torch.tensor(cu, dtype=torch.int32, device=DEV),
                            torch.tensor(lens, dtype=torch.int32, device=DEV), table, tail,
                            max_new=max(call))
        assert api.check_status() == 0
        for s in range(S):
            lens[s] += cu[s + 1] - cu[s]
            if lens[s] > 0:
                _pages_equal(cache, perm[s], *seqs[s], lens[s])
    return cache, table, seqs, lens


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_append_token_by_token_and_chunks(dtype):
    # one token per call across a group and a page boundary, then chunks of 5, 31, 64 and 100
    plan = [[1, 1, 1]] * 70 + [[5, 31, 64], [31, 5, 100], [100, 64, 1], [64, 100, 31]]
    _run(dtype, [300, 290, 260], plan)


def test_append_whole_prompts_then_steps():
    plan = [[777, 129, 64, 1]] + [[1, 1, 1, 1]] * 33
    _run(torch.bfloat16, [810, 162, 97, 34], plan, hkv=3, seed=3)


def test_decode_after_appends_matches_one_piece_cache():
    cache, table, seqs, lens = _run(torch.bfloat16, [520, 333], [[200, 33], [1, 1], [319, 299]],
                                    hkv=2, seed=5)
    ref = paged.empty_cache(cache.k_pages.shape[0], 2, 128, KTS, DEV)
    for s, (k, v) in enumerate(seqs):
        paged.write_sequence(ref, k.to(DEV), v.to(DEV), table[s, :(lens[s] + 63) // 64])
    g = torch.Generator().manual_seed(9)
    q4 = api.quantize_nvfp4(torch.randn(2, 8, 128, generator=g).to(torch.bfloat16).to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    a = api.attn_qk4v8_decode_paged(q4, cache, table, ctx, max(lens), 256, out_dtype=torch.float32)
    b = api.attn_qk4v8_decode_paged(q4, ref, table, ctx, max(lens), 256, out_dtype=torch.float32)
    assert torch.equal(a, b)


def test_append_bad_page_id_reports_bounds_error():
    d, hkv = 128, 1
    cache = paged.empty_cache(4, hkv, d, KTS, DEV)
    tail = paged.empty_tail(1, hkv, d, torch.bfloat16, DEV)
    table = torch.tensor([[0, 9]], dtype=torch.int32, device=DEV)          # page 9 does not exist
    k = torch.randn(100, hkv, d, dtype=torch.bfloat16, device=DEV)
    api.kv_append_paged(cache, k, k.clone(), torch.tensor([0, 100], dtype=torch.int32, device=DEV),
                        torch.tensor([0], dtype=torch.int32, device=DEV), table, tail, max_new=100)
    assert api.check_status() == 5
    assert not cache.k_pages[1:].any()                                       # nothing stray
