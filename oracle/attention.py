"""Oracle — QK4V8 attention, FP16 tiles, paged split-K decode (TEST INFRASTRUCTURE ONLY).

Plain float64 restatement of the method, one (batch, query head) at a time, key tiles of 128
in ascending order. Sources:

* FlashAttention tiling with an online softmax kept in high precision: hotelren.com MpFA
  article §3.3 ("online softmax", running max and running sum in FP32, never FP16) and §3.4
  (tiling); §1 (fused kernel, QK 4-bit / V 8-bit).
* Block-scaled products with the scales folded in afterwards: zdszero primer, "GEMM 的通用形式"
  (Y ≈ (Q_X Q_W)(s_X s_W)).
* P quantized to E4M3 before the PV product ("fused probability quantization"):
  sns.style BitDecoding-FP4 summary, system-level techniques; the P*448 scaling per 128-key
  tile is the problem statement's.
* Selected tiles in FP16 merged through the same online softmax: ai-feeds.com ThriftAttention
  summary, "方法" step 3.
* Paged KV cache read once per decoding step, GQA: sns.style BitDecoding-FP4 summary.

Per query row i, with x_hat the float64 dequantized operands:

    m = -inf, l = 0, O = 0
    for each key tile t = 0, 1, ... (keys j masked when causal and j > i, or j >= Nk):
        s_j   = (q_hat_i . k_hat_j) * softmax_scale
        m_new = max(m, max_j s_j)                 (a row with every key masked is skipped)
        p~_j  = exp(s_j - m_new)                 in [0, 1]
        p_j   = decode_E4M3(E4M3(448 p~_j)) / 448
        alpha = exp(m - m_new);  l = alpha l + sum_j p_j;  O = alpha O + sum_j p_j v_hat_j
        m     = m_new
    O_i = O / l

Readings (the pages are silent on each): l sums the quantized p, so constant V gives O equal
to that constant and the weights sum to one exactly; P is encoded against the running max
after the tile is included; no clipping of QK^T; causal means j <= i with Nq == Nk.

FP16 tile (a tile marked in the selection): s_j from the 16-bit inputs as given (fp16 or bf16
values; a 16-bit tensor core multiplies either exactly, so the page's "FP16" is read as the
16-bit precision of the inputs, not a re-rounding of bf16 Q and K to fp16), and
p_j = fp16(448 p~_j) / 448 (the FP16 branch works in the same P*448 units as the E4M3
branch, so both accumulate into one O); V from its FP16-rounded copy (P and V meet in one
FP16 product).

Underflow-aware probability scaling (sns.style BitDecoding-FP4 summary, the second algorithm
item: long-context probabilities are tiny, the E4M3 encoding of P can round whole blocks to
zero, so the probability scaling is adjusted to avoid it). Reading (the page gives no formula):
each 32-key block b of a tile row gets its own power-of-two scale 2^e_b, e_b = ceil(log2 of
the block's largest p~) clipped to [-127, 0] (0 for an all-zero block), and

    p_j = decode_E4M3(E4M3(448 p~_j 2^-e_b)) 2^e_b / 448

so every block's largest value lands in (224, 448] before rounding. This is the E8M0 block
scale the FP8 MMA applies to its P operand; l and O see the same p_j.

Split-K decode: the key range of a sequence is cut into splits of ``split_tokens`` keys
(a multiple of 128; 0 means one split). Each split runs the loop above from m = -inf, and the
splits merge exactly: M = max_s m_s, O = sum_s e^(m_s - M) O_s / sum_s e^(m_s - M) l_s.
"""
from __future__ import annotations

import numpy as np

from .formats import e4m3_round, fp16_round

TILE = 128
P_SCALE = 448.0


def _p_e4m3(p_tilde: np.ndarray) -> np.ndarray:
    return e4m3_round(p_tilde * P_SCALE) / P_SCALE


def _p_fp16(p_tilde: np.ndarray) -> np.ndarray:
    return fp16_round(p_tilde * P_SCALE) / P_SCALE


def _p_e4m3_block_scaled(p_tilde: np.ndarray) -> np.ndarray:
    """Underflow-aware P: per row and 32-key block, scale by 2^-e_b before the E4M3 encode."""
    p = np.zeros_like(p_tilde)
    for b in range(0, p_tilde.shape[1], 32):
        blk = p_tilde[:, b:b + 32]
        mx = blk.max(axis=1)
        e = np.zeros(mx.shape)
        pos = mx > 0
        e[pos] = np.clip(np.ceil(np.log2(mx[pos])), -127, 0)
        sc = np.ldexp(1.0, e.astype(np.int64))[:, None]
        p[:, b:b + 32] = e4m3_round(blk * P_SCALE / sc) * sc / P_SCALE
    return p


def attention_rows(q: np.ndarray, row_pos: np.ndarray, k: np.ndarray, v: np.ndarray,
                   causal: bool, softmax_scale: float, *,
                   quantize_p: bool = True, p_underflow_aware: bool = False,
                   fp16_select=None, q16=None, k16=None, v16=None,
                   key_begin: int = 0, key_end: int | None = None):
    """Online-softmax attention of query rows ``q`` [R, d] at positions ``row_pos`` over keys
    ``k``/``v`` [Nk, d] restricted to [key_begin, key_end) in 128-key tiles (tile t covers
    keys [128 t, 128 t + 128)).

    ``fp16_select(q_tile_of_rows [R], t) -> bool [R]`` marks rows whose (query tile, key
    tile) pair takes the FP16 branch; q16/k16/v16 are then that branch's operands (Q and K as
    given, V rounded to FP16).
    Returns the un-normalised state (m, l, O) in float64.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    row_pos = np.asarray(row_pos, dtype=np.int64)
    r, d = q.shape
    nk = k.shape[0] if key_end is None else key_end
    m = np.full(r, -np.inf)
    l = np.zeros(r)
    o = np.zeros((r, d))
    q_tile = row_pos // TILE
    t_begin = key_begin // TILE
    t_end = (nk + TILE - 1) // TILE
    for t in range(t_begin, t_end):
        j0, j1 = t * TILE, min((t + 1) * TILE, nk)
        keys = np.arange(j0, j1)
        # rows with at least one visible key in this tile; the others keep their state
        rows = np.nonzero(row_pos >= j0)[0] if causal else np.arange(r)
        if rows.size == 0:
            continue
        valid = np.ones((rows.size, j1 - j0), dtype=bool)
        if causal:
            valid &= keys[None, :] <= row_pos[rows, None]
        s = (q[rows] @ k[j0:j1].T) * softmax_scale
        sel = np.zeros(rows.size, dtype=bool) if fp16_select is None else fp16_select(q_tile[rows], t)
        if sel.any():
            s[sel] = (q16[rows[sel]] @ k16[j0:j1].T) * softmax_scale
        s = np.where(valid, s, -np.inf)
        m_old = m[rows]
        m_new = np.maximum(m_old, s.max(axis=1))
        p_tilde = np.where(valid, np.exp(s - m_new[:, None]), 0.0)
        if quantize_p:
            p = _p_e4m3_block_scaled(p_tilde) if p_underflow_aware else _p_e4m3(p_tilde)
            if sel.any():
                p[sel] = _p_fp16(p_tilde[sel])
        else:
            p = p_tilde
        alpha = np.where(np.isfinite(m_old), np.exp(np.where(np.isfinite(m_old), m_old, 0.0) - m_new), 0.0)
        pv = p @ v[j0:j1]
        if sel.any():
            pv[sel] = p[sel] @ v16[j0:j1]
        l[rows] = alpha * l[rows] + p.sum(axis=1)
        o[rows] = alpha[:, None] * o[rows] + pv
        m[rows] = m_new
    return m, l, o


def finish(m: np.ndarray, l: np.ndarray, o: np.ndarray):
    """Normalise: O / l, and the natural-log LSE m + ln l."""
    with np.errstate(divide="ignore", invalid="ignore"):
        out = o / l[:, None]
        lse = m + np.log(l)
    return out, lse


def merge_splits(parts):
    """Exact merge of split states [(m, l, O), ...] of the same rows."""
    ms = np.stack([p[0] for p in parts])
    big_m = ms.max(axis=0)
    safe = np.where(np.isfinite(big_m), big_m, 0.0)
    w = np.where(np.isfinite(ms), np.exp(np.where(np.isfinite(ms), ms, 0.0) - safe), 0.0)
    l = sum(w[i] * parts[i][1] for i in range(len(parts)))
    o = sum(w[i][:, None] * parts[i][2] for i in range(len(parts)))
    return big_m, l, o


def attention_head(q, k, v, causal, softmax_scale, **kw):
    """All rows of one (batch, query head): q [Nq, d], k/v [Nk, d]; returns (O, lse)."""
    rows = np.arange(q.shape[0])
    m, l, o = attention_rows(q, rows, k, v, causal, softmax_scale, **kw)
    return finish(m, l, o)


def exact_attention(q, k, v, causal, softmax_scale):
    """Textbook softmax(q k^T * scale) v in float64, no tiling (the brute-force pin)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    s = (q @ k.T) * softmax_scale
    if causal:
        nq, nk = s.shape
        s = np.where(np.arange(nk)[None, :] <= np.arange(nq)[:, None], s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def decode_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, length: int,
                softmax_scale: float, split_tokens: int, p_underflow_aware: bool = False):
    """One decode step for the query rows ``q`` [R, d] of one sequence over its first
    ``length`` keys, in splits of ``split_tokens`` keys (0: one split). Returns (O, lse)."""
    if split_tokens <= 0:
        split_tokens = max(length, 1)
    assert split_tokens % TILE == 0 or split_tokens >= length
    rows = np.full(q.shape[0], length - 1)
    parts = []
    for b in range(0, length, split_tokens):
        parts.append(attention_rows(q, rows, k, v, False, softmax_scale,
                                    p_underflow_aware=p_underflow_aware,
                                    key_begin=b, key_end=min(b + split_tokens, length)))
    return finish(*merge_splits(parts))
