"""Oracle — tile importance scores and top-fraction selection (TEST INFRASTRUCTURE ONLY).

Source: ai-feeds.com ThriftAttention summary, "方法" step 2 (score every 128x128 query-key
tile with a cheap estimate of the tile's largest attention weight, from partial products or
norms; keep about the top 5 %) and "局限" (the score is an L2-norm bound of the query-key
product).

Reading: the Cauchy-Schwarz bound  max_{i in Q tile} |q_hat_i| * max_{j in K tile} |k_hat_j|,
computed exactly in integers from the NVFP4 codes. With E2M1 magnitudes doubled to integers
{0,1,2,3,4,6,8,12} and E4M3 scale values times 2^9 (integers up to 229376),

    N_r = sum_blocks (2^9 s_b)^2 * sum_{e in block} (2 e)^2  =  |x_hat_r|^2 * 2^20 / s_t^2,

an exact integer below 2^51. The tile score is max N_r(q) * max N_r(k) (below 2^102, exact
as a Python int). The per-tensor scales are common to every tile of a head and do not change
the ranking.

Candidates: every tile pair that is not fully masked (causal: k_tile <= q_tile). The number
kept per (batch, query head) is ceil(n_candidates * frac_bp / 10000) (the fraction in basis
points, so the count is exact). Ranking: higher score first, then the lower linear index
q_tile * T_k + k_tile.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e4m3_decode
from .quant import NVFP4_BLOCK, nvfp4_unpack

TILE = 128


def row_norms_int(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Exact N_r for rows of NVFP4 codes: packed [rows, d/2], scales [rows, d/16] -> int64."""
    codes = nvfp4_unpack(packed)
    e2 = np.rint(2.0 * np.abs(e2m1_decode(codes))).astype(np.int64)          # {0..12}
    rows, d = e2.shape
    blk = (e2 * e2).reshape(rows, d // NVFP4_BLOCK, NVFP4_BLOCK).sum(axis=2)   # <= 2304
    sb = np.rint(e4m3_decode(scales) * 512.0).astype(np.int64)                 # <= 229376
    return (sb * sb * blk).sum(axis=1)


def tile_max(norms: np.ndarray, n: int) -> list[int]:
    t = (n + TILE - 1) // TILE
    return [int(norms[i * TILE:min((i + 1) * TILE, n)].max()) for i in range(t)]


def n_select(n_candidates: int, frac_bp: int) -> int:
    return (n_candidates * frac_bp + 9999) // 10000


def select_tiles(q_norms: np.ndarray, k_norms: np.ndarray, nq: int, nk: int,
                 causal: bool, frac_bp: int):
    """Ranked selection for one (batch, query head).

    Returns (idx list of q_tile * T_k + k_tile in rank order, bitmap uint8 [T_q, T_k]).
    """
    mq = tile_max(q_norms, nq)
    mk = tile_max(k_norms, nk)
    tq, tk = len(mq), len(mk)
    cand = []
    for qt in range(tq):
        for kt in range(tk):
            if causal and kt > qt:
                continue
            cand.append((-(mq[qt] * mk[kt]), qt * tk + kt))
    cand.sort()
    keep = n_select(len(cand), frac_bp)
    idx = [c[1] for c in cand[:keep]]
    bitmap = np.zeros((tq, tk), dtype=np.uint8)
    for i in idx:
        bitmap[i // tk, i % tk] = 1
    return idx, bitmap


def tile_scores(q_norms, k_norms, nq, nk):
    """All tile scores as Python ints, [T_q][T_k] (for tests)."""
    mq = tile_max(q_norms, nq)
    mk = tile_max(k_norms, nk)
    return [[a * b for b in mk] for a in mq]
