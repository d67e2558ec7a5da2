"""Pins for oracle/tilescore.py: the exact integer norm against the float64 norm of the
dequantized rows (closed form), brute-force ranking on tiny inputs, counts and tie-breaks."""
import numpy as np
import pytest

from oracle import quant as Q
from oracle import tilescore as T


def test_row_norm_closed_form():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((300, 128)) * 5).astype(np.float32)
    codes, scales, s_t = Q.nvfp4_quantize(x)
    n_int = T.row_norms_int(codes, scales)
    xh = Q.nvfp4_dequantize(codes, scales, s_t)
    n_flt = (xh ** 2).sum(axis=1) * 2.0 ** 20 / np.float64(s_t) ** 2
    assert np.allclose(n_int, n_flt, rtol=1e-12, atol=0)
    assert n_int.max() < 2 ** 51


def test_counts_match_problem_sizes():
    # 16384 tokens, causal: T = 128, T(T+1)/2 = 8256 candidates, 5 % -> 413
    assert 128 * 129 // 2 == 8256
    assert T.n_select(8256, 500) == 413
    assert T.n_select(100, 500) == 5 and T.n_select(101, 500) == 6 and T.n_select(0, 500) == 0


@pytest.mark.parametrize("causal", [False, True])
def test_selection_matches_brute_force_float_ranking(causal):
    rng = np.random.default_rng(1)
    n = 700                                             # 6 tiles, ragged last tile
    q = (rng.standard_normal((n, 64)) * rng.uniform(0.2, 3, (n, 1))).astype(np.float32)
    k = (rng.standard_normal((n, 64)) * rng.uniform(0.2, 3, (n, 1))).astype(np.float32)
    qc, qs, qt = Q.nvfp4_quantize(q)
    kc, ks, kt = Q.nvfp4_quantize(k)
    idx, bitmap = T.select_tiles(T.row_norms_int(qc, qs), T.row_norms_int(kc, ks), n, n,
                                 causal, 2500)
    # brute force: float64 norms of the dequantized rows, all pairs, sort
    qn = np.linalg.norm(Q.nvfp4_dequantize(qc, qs, qt), axis=1)
    kn = np.linalg.norm(Q.nvfp4_dequantize(kc, ks, kt), axis=1)
    tiles = 6
    sc = []
    for a in range(tiles):
        for b in range(tiles):
            if causal and b > a:
                continue
            s = qn[a * 128:(a + 1) * 128].max() * kn[b * 128:(b + 1) * 128].max()
            sc.append((-s, a * tiles + b))
    sc.sort()
    want = [i for _, i in sc[:T.n_select(len(sc), 2500)]]
    assert idx == want
    assert bitmap.sum() == len(want)
    for i in want:
        assert bitmap[i // tiles, i % tiles] == 1


def test_tie_break_lower_index_first():
    qn = np.array([5] * 128 + [5] * 128, dtype=np.int64)
    kn = np.array([3] * 128 + [3] * 128, dtype=np.int64)
    idx, _ = T.select_tiles(qn, kn, 256, 256, False, 5000)
    assert idx == [0, 1]
    kn2 = kn.copy(); kn2[200] = 4
    idx, _ = T.select_tiles(qn, kn2, 256, 256, True, 10000)
    assert idx == [1 * 2 + 1, 0, 2]        # (1,1) has the larger K tile max, then ties by index


def test_scores_are_products_of_tile_maxima():
    qn = np.arange(300, dtype=np.int64) * 7
    kn = (np.arange(300, dtype=np.int64) % 50) + 1
    s = T.tile_scores(qn, kn, 300, 300)
    assert s[2][0] == qn[256:300].max() * kn[:128].max()
    assert s[1][2] == qn[128:256].max() * kn[256:300].max()
