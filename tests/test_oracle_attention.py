"""Pins for oracle/attention.py: brute-force exact attention, hand-worked examples, and the
invariants the method fixes (constant V, first causal row, weights sum to one, V * 2^k)."""
import math

import numpy as np
import pytest

from oracle import attention as A
from oracle import formats as F
from oracle import quant as Q
from golden_io import keyed


def _rand(seed, nq, nk, d, scale_k=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((nq, d))
    k = rng.standard_normal((nk, d)) * scale_k
    v = rng.standard_normal((nk, d))
    return q, k, v


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n", [1, 100, 128, 129, 300])
def test_tiled_online_softmax_equals_exact_attention(causal, n):
    q, k, v = _rand(n, n, n, 32, scale_k=2.0)
    o, _ = A.attention_head(q, k, v, causal, 1 / math.sqrt(32), quantize_p=False)
    ref = A.exact_attention(q, k, v, causal, 1 / math.sqrt(32))
    assert np.max(np.abs(o - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_hand_worked_examples():
    g = keyed("attention_examples.txt")
    d = 64
    q = np.zeros((1, d)); q[0, 0] = 8.0
    # example A
    k = np.zeros((2, d)); k[1, 0] = -1.0
    v = np.zeros((2, d)); v[0, 0] = 1.0; v[1, 1] = 1.0
    o, _ = A.attention_head(q, k, v, False, 1 / 8)
    want = [float(t) for t in g["A"]]
    assert np.allclose(o[0, :3], want, rtol=0, atol=1e-15)
    # example B
    k = np.zeros((129, d)); k[1:128, 0] = -100.0; k[128, 0] = 2.0
    v = np.zeros((129, d)); v[:, 2] = 1.0; v[0] = 0; v[0, 0] = 1.0; v[128] = 0; v[128, 1] = 1.0
    o, _ = A.attention_head(q, k, v, False, 1 / 8)
    want = [float(t) for t in g["B"]]
    assert np.allclose(o[0, :3], want, rtol=0, atol=1e-15)


def test_hand_worked_underflow_aware_example():
    g = keyed("attention_examples.txt")
    d = 64
    q = np.zeros((1, d)); q[0, 0] = 8.0
    k = np.zeros((64, d)); k[:, 0] = -100.0; k[0, 0] = 0.0; k[32, 0] = -12.0
    v = np.zeros((64, d)); v[:, 2] = 1.0
    v[0] = 0; v[0, 0] = 1.0; v[32] = 0; v[32, 1] = 1.0
    o, _ = A.attention_head(q, k, v, False, 1 / 8, p_underflow_aware=True)
    assert np.allclose(o[0, :3], [float(t) for t in g["E"]], rtol=0, atol=1e-15)
    o_fixed, _ = A.attention_head(q, k, v, False, 1 / 8)
    assert abs(o_fixed[0, 1] - float(g["E"][1])) > 1e-6       # the fixed encoding differs


def test_hand_worked_split_decode_examples():
    g = keyed("attention_examples.txt")
    d = 64
    q = np.zeros((1, d)); q[0, 0] = 8.0
    k = np.zeros((256, d)); k[:, 0] = -100.0; k[0, 0] = 2.0; k[128, 0] = 0.0; k[129, 0] = -1.0
    v = np.zeros((256, d)); v[:, 2] = 1.0
    for j, c in ((0, 0), (128, 1), (129, 3)):
        v[j] = 0; v[j, c] = 1.0
    for key, split in (("F", 128), ("G", 256)):
        o, _ = A.decode_rows(q, k, v, 256, 1 / 8, split)
        assert np.allclose(o[0, :4], [float(t) for t in g[key]], rtol=0, atol=1e-15), key


def test_hand_worked_fp16_tile_examples():
    g = keyed("attention_examples.txt")
    d = 64
    q = np.zeros((1, d)); q[0, 0] = 8.0
    # example C: example A's single tile in FP16 (operands exact in fp16)
    k = np.zeros((2, d)); k[1, 0] = -1.0
    v = np.zeros((2, d)); v[0, 0] = 1.0; v[1, 1] = 1.0
    every = lambda qt, t: np.ones(qt.shape, dtype=bool)
    o, _ = A.attention_head(q, k, v, False, 1 / 8, fp16_select=every, q16=q, k16=k, v16=v)
    assert np.allclose(o[0, :3], [float(t) for t in g["C"]], rtol=0, atol=1e-15)
    # example D: tile 0 in E4M3, tile 1 in FP16 with a rise of the running max
    k = np.zeros((130, d)); k[1:128, 0] = -100.0; k[128, 0] = 2.0; k[129, 0] = 1.0
    v = np.zeros((130, d)); v[:, 2] = 1.0
    v[0] = 0; v[0, 0] = 1.0; v[128] = 0; v[128, 1] = 1.0; v[129] = 0; v[129, 3] = 1.0
    second = lambda qt, t: np.full(qt.shape, t == 1)
    o, _ = A.attention_head(q, k, v, False, 1 / 8, fp16_select=second, q16=q, k16=k, v16=v)
    assert np.allclose(o[0, :4], [float(t) for t in g["D"]], rtol=0, atol=1e-15)


@pytest.mark.parametrize("c", [1.0, 0.375, -2.5])
def test_constant_v_gives_constant_output(c):
    q, k, _ = _rand(4, 200, 200, 64, scale_k=3.0)
    v = np.full((200, 64), c)
    for causal in (False, True):
        o, _ = A.attention_head(q, k, v, causal, 0.125)
        assert np.max(np.abs(o - c)) <= 1e-13 * abs(c)


def test_first_causal_row_is_v0():
    q, k, v = _rand(5, 130, 130, 64)
    o, _ = A.attention_head(q, k, v, True, 0.125)
    assert np.array_equal(o[0], v[0])


def test_weights_sum_to_one_and_are_e4m3_multiples():
    """With V = identity, O's row is the weight vector p / l: it sums to one, and l * O is a
    vector of E4M3 values / 448 (per tile, up to the alpha rescale of earlier tiles)."""
    n = 100
    q, k, _ = _rand(6, 3, n, 128, scale_k=2.0)
    v = np.eye(n, 128)
    m, l, o = A.attention_rows(q, np.arange(3), k, v, False, 0.1)
    w = o / l[:, None]
    assert np.allclose(w.sum(axis=1), 1.0, atol=1e-14)
    codes = o * 448.0                              # one tile: no rescale
    assert np.array_equal(F.e4m3_round(codes), codes)


@pytest.mark.parametrize("kexp", [-3, 5])
def test_v_power_of_two_scaling(kexp):
    q, k, v = _rand(8, 150, 150, 64, scale_k=2.0)
    o0, _ = A.attention_head(q, k, v, True, 0.125)
    o1, _ = A.attention_head(q, k, v * 2.0 ** kexp, True, 0.125)
    assert np.array_equal(o1, o0 * 2.0 ** kexp)


def test_p_quantization_error_is_bounded():
    """E4M3 rounds each weight by at most 2^-4 relative (or 2^-10/448 absolute), so O moves by
    at most ~2 * 2^-4 * max|v| from exact attention on the same dequantized operands."""
    q, k, v = _rand(9, 256, 256, 64, scale_k=2.0)
    o, _ = A.attention_head(q, k, v, True, 0.125)
    ref = A.exact_attention(q, k, v, True, 0.125)
    assert np.max(np.abs(o - ref)) <= 2 * 2.0 ** -4 * np.abs(v).max()
    assert np.max(np.abs(o - ref)) > 0                  # the quantization is really applied


def test_quantized_operands_close_to_unquantized():
    """Full QK4V8 pipeline on quantized operands stays near exact float attention (a quality
    figure; the bound here only guards against a grossly wrong dequantization)."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((3, 256, 64)).astype(np.float32)
    qc, qs, qt = Q.nvfp4_quantize(x[0])
    kc, ks, kt = Q.nvfp4_quantize(x[1])
    vc, vs = Q.mxfp8_quantize_v(x[2])
    qh = Q.nvfp4_dequantize(qc, qs, qt)
    kh = Q.nvfp4_dequantize(kc, ks, kt)
    vh = Q.mxfp8_dequantize_v(vc, vs, 256)
    o, _ = A.attention_head(qh, kh, vh, True, 0.125)
    ref = A.exact_attention(x[0], x[1], x[2], True, 0.125)
    rel = np.sqrt(np.mean((o - ref) ** 2)) / np.sqrt(np.mean(ref ** 2))
    assert rel < 0.15


def test_fp16_tiles_everywhere_close_to_exact_on_fp16_operands():
    q, k, v = _rand(10, 200, 200, 64, scale_k=2.0)
    q16, k16, v16 = (F.fp16_round(t) for t in (q, k, v))
    sel_all = lambda qt, t: np.ones(qt.shape, dtype=bool)
    m, l, o = A.attention_rows(q, np.arange(200), k, v, True, 0.125,
                               fp16_select=sel_all, q16=q16, k16=k16, v16=v16)
    out, _ = A.finish(m, l, o)
    ref = A.exact_attention(q16, k16, v16, True, 0.125)
    # only the fp16 rounding of 448 p~ remains: 2^-11 relative per weight
    assert np.max(np.abs(out - ref)) <= 2 * 2.0 ** -11 * np.abs(v16).max()
    # and without P rounding it is exact attention on the fp16 operands
    m, l, o = A.attention_rows(q, np.arange(200), k, v, True, 0.125, quantize_p=False,
                               fp16_select=sel_all, q16=q16, k16=k16, v16=v16)
    out, _ = A.finish(m, l, o)
    assert np.max(np.abs(out - ref)) <= 1e-12


def test_fp16_selection_only_changes_selected_tiles():
    q, k, v = _rand(11, 256, 256, 64, scale_k=2.0)
    q16, k16, v16 = (F.fp16_round(t) for t in (q, k, v))
    none = lambda qt, t: np.zeros(qt.shape, dtype=bool)
    base = A.attention_rows(q, np.arange(256), k, v, True, 0.125)
    same = A.attention_rows(q, np.arange(256), k, v, True, 0.125,
                            fp16_select=none, q16=q16, k16=k16, v16=v16)
    assert all(np.array_equal(a, b) for a, b in zip(base, same))
    only = lambda qt, t: (qt == 1) & (t == 0)
    mix = A.attention_rows(q, np.arange(256), k, v, True, 0.125,
                           fp16_select=only, q16=q16, k16=k16, v16=v16)
    assert np.array_equal(mix[2][:128], base[2][:128])        # q tile 0 untouched
    assert not np.array_equal(mix[2][128:], base[2][128:])


def test_split_merge_is_exact_without_p_rounding():
    q, k, v = _rand(12, 4, 1000, 64, scale_k=2.0)
    rows = np.full(4, 999)
    parts = [A.attention_rows(q, rows, k, v, False, 0.125, quantize_p=False,
                              key_begin=b, key_end=min(b + 256, 1000)) for b in range(0, 1000, 256)]
    o, _ = A.finish(*A.merge_splits(parts))
    ref = A.exact_attention(q, k, v, False, 0.125)
    assert np.max(np.abs(o - ref)) <= 1e-12


def test_decode_one_split_equals_prefill_row():
    q, k, v = _rand(13, 4, 777, 64, scale_k=2.0)
    o1, _ = A.decode_rows(q, k, v, 777, 0.125, split_tokens=0)
    m, l, o = A.attention_rows(q, np.full(4, 776), k, v, False, 0.125)
    o2, _ = A.finish(m, l, o)
    assert np.array_equal(o1, o2)
    o3, _ = A.decode_rows(q, k, v, 777, 0.125, split_tokens=256)   # splits: close, not equal
    assert np.max(np.abs(o3 - o1)) < 0.1 * np.abs(o1).max()


def test_decode_context_length_one_is_v0():
    q, k, v = _rand(14, 4, 10, 64)
    o, _ = A.decode_rows(q, k, v, 1, 0.125, split_tokens=128)
    assert np.array_equal(o, np.repeat(v[:1], 4, axis=0))


# ---- underflow-aware probability scaling (per 32-key block power-of-two scale) ----

def test_block_scaled_p_relative_error_and_no_block_underflow():
    """Closed form: after the per-block scale every value at or above 2^-6 of its block's
    largest lies in the normal E4M3 range, so its relative error is at most 2^-4; a block
    whose values are all below 2^-10 / 448 encodes to zero with the fixed 448 scale but not
    with the block scale."""
    rng = np.random.default_rng(3)
    p = np.exp2(rng.uniform(-40, 0, (64, 128)))
    p[:, 32:64] *= 2.0 ** -30                            # a whole block far below the row max
    got = A._p_e4m3_block_scaled(p)
    for b in range(0, 128, 32):
        blk, g = p[:, b:b + 32], got[:, b:b + 32]
        big = blk >= blk.max(axis=1, keepdims=True) * 2.0 ** -6
        assert np.all(np.abs(g[big] - blk[big]) <= blk[big] * 2.0 ** -4)
        assert np.all(g.max(axis=1) > 0)
    tiny = p[:, 32:64].max(axis=1) < 2.0 ** -10 / 448
    assert tiny.any()
    assert np.all(A._p_e4m3(p[tiny, 32:64]) == 0)
    assert np.all(got[tiny, 32:64].max(axis=1) > 0)


def test_block_scaled_p_equals_fixed_when_every_block_holds_a_top_value():
    """A block whose largest p~ is above 1/2 gets e_b = 0: the encoding is the fixed one."""
    rng = np.random.default_rng(4)
    p = rng.uniform(0, 1, (16, 128))
    p[:, ::32] = rng.uniform(0.51, 1.0, (16, 4))
    assert np.array_equal(A._p_e4m3_block_scaled(p), A._p_e4m3(p))


def test_underflow_aware_constant_v_and_closer_to_exact():
    """Constant V still gives exactly that constant (l and O see the same p). One key 14 nats
    above 4095 others: each of those has p~ = e^-14 < 2^-10 / 448, so the fixed scale drops
    them all (O = the top key's v) although together they hold 4095 e^-14 = 0.34 % of the
    weight; the block scale keeps them and lands within E4M3 precision of the exact result."""
    d, n, scale = 16, 4096, 0.25
    q = np.zeros((1, d)); q[0, 0] = 1.0
    k = np.zeros((n, d)); k[:, 0] = 6.0 / scale; k[5, 0] = 20.0 / scale
    v = np.full((n, d), 0.75)
    o, _ = A.decode_rows(q, k, v, n, scale, 0, p_underflow_aware=True)
    assert np.allclose(o, 0.75, rtol=0, atol=1e-12)
    rng = np.random.default_rng(5)
    v = rng.standard_normal((n, d)) + 3.0
    ref = A.exact_attention(q, k, v, False, scale)
    o_fix, _ = A.decode_rows(q, k, v, n, scale, 0)
    o_ua, _ = A.decode_rows(q, k, v, n, scale, 0, p_underflow_aware=True)
    assert np.array_equal(o_fix[0], v[5])                      # every other key dropped
    err_fix = np.abs(o_fix - ref).max()
    err_ua = np.abs(o_ua - ref).max()
    assert err_fix > 5e-3 and err_ua < err_fix / 20
