"""GPU parity of the tile scorer (bit-exact selection) and of the FP16-tile attention path."""
import math

import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, workloads
from oracle import quant as OQ
from oracle import tilescore as OT
from helpers import assert_attention_close, f32, oracle_prefill_rows, oracle_tensor_scale

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_norms(x, s_t):
    """Exact row norms of every head of x [B, H, N, D], quantized with tensor scale s_t."""
    B, H, N, D = x.shape
    out = np.zeros((B, H, N), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            c, s, _ = OQ.nvfp4_quantize(f32(x[b, h]), tensor_scale=s_t)
            out[b, h] = OT.row_norms_int(c, s)
    return out


def _check_selection(q, k, causal, frac_bp, heads=None):
    """Tile selection of the GPU against the oracle's, bit for bit, on the given query heads
    (all by default). Returns the oracle's bitmaps {(b, hq): [T, T]} for those heads."""
    q4, k4 = api.quantize_nvfp4(q.to(DEV)), api.quantize_nvfp4(k.to(DEV))
    idx, n_sel, bitmap = api.tile_score_select(q4, k4, causal, frac_bp)
    B, Hq, N, _ = q.shape
    Hkv = k.shape[1]
    qn = _oracle_norms(q, oracle_tensor_scale(q))
    kn = _oracle_norms(k, oracle_tensor_scale(k))
    idx, n_sel, bitmap = idx.cpu().numpy(), n_sel.cpu().numpy(), bitmap.cpu().numpy()
    oracle_bm = {}
    for b in range(B):
        for hq in (range(Hq) if heads is None else heads):
            want, wbm = OT.select_tiles(qn[b, hq], kn[b, hq // (Hq // Hkv)], N, N, causal, frac_bp)
            bh = b * Hq + hq
            assert n_sel[bh] == len(want)
            assert idx[bh, :len(want)].tolist() == want, (b, hq)
            assert np.array_equal(bitmap[bh], wbm)
            oracle_bm[(b, hq)] = wbm
    return oracle_bm


@pytest.mark.parametrize("N,causal,frac", [(1000, True, 2500), (700, False, 500), (128, True, 10000),
                                           (3000, True, 500)])
def test_tile_selection_bit_exact(N, causal, frac):
    g = torch.Generator().manual_seed(N)
    q = (torch.randn(2, 4, N, 128, generator=g) * torch.rand(2, 4, N, 1, generator=g) * 3).to(torch.bfloat16)
    k = (torch.randn(2, 2, N, 128, generator=g) * torch.rand(2, 2, N, 1, generator=g) * 3).to(torch.bfloat16)
    _check_selection(q, k, causal, frac)


def test_tile_selection_ties_take_lower_index():
    q = torch.ones(1, 1, 512, 64, dtype=torch.bfloat16)
    k = torch.ones(1, 1, 512, 64, dtype=torch.bfloat16)
    _check_selection(q, k, True, 3000)


def test_mixed_workload_selection_and_sampled_attention():
    """The 16K selective workload: the GPU's tile selection equals the oracle's on the sampled
    heads, and attention (which selects again inside qk4v8_attention) matches the oracle run
    with the oracle's own selection."""
    w = workloads.make_prefill("mixed_prefill_n16384")
    N, scale = 16384, 1 / math.sqrt(128)
    rng = np.random.default_rng(3)
    heads = sorted(rng.choice(32, size=2, replace=False).tolist())
    oracle_bm = _check_selection(w.q, w.k, True, 500, heads=heads)
    out = api.qk4v8_attention(w.q.to(DEV), w.k.to(DEV), w.v.to(DEV), True, scale, fp16_frac_bp=500,
                              out_dtype=torch.float32)
    got, want = [], []
    for hq in heads:
        bm = oracle_bm[(0, hq)]
        sel_qt = np.nonzero(bm.any(axis=1))[0]
        # at least half the rows from query tiles that hold a selected tile
        r1 = rng.choice(sel_qt, size=128) * 128 + rng.integers(0, 128, size=128)
        r2 = rng.choice(N, size=128, replace=False)
        rows = np.unique(np.concatenate([r1, r2]))
        sel = lambda qt, t, bm=bm: bm[qt, t].astype(bool)
        o, _ = oracle_prefill_rows(w.q, w.k, w.v, hq, rows, True, scale, fp16_select=sel)
        want.append(o)
        got.append(f32(out[0, hq, torch.as_tensor(rows, device=DEV)]))
    assert_attention_close(np.concatenate(got), np.concatenate(want), "mixed 16k sampled")


@pytest.mark.parametrize("frac", [2500, 10000])
def test_mixed_small_full(frac):
    """Every head and row: the GPU's selection equals the oracle's, and attention matches the
    oracle run with the oracle's selection."""
    g = torch.Generator().manual_seed(frac)
    q = torch.randn(1, 4, 600, 128, generator=g).to(torch.bfloat16)
    k = (torch.randn(1, 2, 600, 128, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(1, 2, 600, 128, generator=g).to(torch.bfloat16)
    oracle_bm = _check_selection(q, k, True, frac)
    out = api.qk4v8_attention(q.to(DEV), k.to(DEV), v.to(DEV), True, fp16_frac_bp=frac,
                              out_dtype=torch.float32)
    got, want = [], []
    for hq in range(4):
        bm = oracle_bm[(0, hq)]
        sel = lambda qt, t, bm=bm: bm[qt, t].astype(bool)
        o, _ = oracle_prefill_rows(q, k, v, hq, np.arange(600), True, 1 / math.sqrt(128), fp16_select=sel)
        want.append(o)
        got.append(f32(out[0, hq]))
    assert_attention_close(np.concatenate(got), np.concatenate(want), f"mixed {frac}")
