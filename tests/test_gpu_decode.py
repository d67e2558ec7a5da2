"""GPU parity of the paged split-K decode against the oracle, page-permutation invariance,
and the device-side page-id bounds check."""
import math

import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, paged, workloads
from oracle import attention as OA
from oracle import quant as OQ
from oracle import paged as OP
from helpers import assert_attention_close, f32, oracle_tensor_scale

pytestmark = pytest.mark.gpu
DEV = "cuda"
KTS = workloads.DECODE_K_TENSOR_SCALE


def _build(lens, hkv, d, seed, shuffle=True):
    g = torch.Generator().manual_seed(seed)
    pages_per = [(n + 63) // 64 for n in lens]
    total = sum(pages_per)
    perm = torch.randperm(total, generator=g)
    if not shuffle:
        perm = torch.arange(total)
    table = torch.full((len(lens), max(pages_per)), -1, dtype=torch.int32)
    seqs, off = [], 0
    cache = paged.empty_cache(total, hkv, d, KTS, DEV)
    for s, n in enumerate(lens):
        table[s, :pages_per[s]] = perm[off:off + pages_per[s]].int()
        off += pages_per[s]
        k = ((torch.randn(n, hkv, d, generator=g) + 0.3) * 3).to(torch.bfloat16)
        v = torch.randn(n, hkv, d, generator=g).to(torch.bfloat16)
        seqs.append((k, v))
        paged.write_sequence(cache, k.to(DEV), v.to(DEV), table[s, :pages_per[s]])
    return cache, table, seqs


def _oracle_decode(q, seqs, lens, hq, hkv, split, scale, ua=False, exact=False, dual=False):
    """Oracle outputs [S, Hq, D] from the dense per-sequence K/V and the step's q."""
    S, _, d = q.shape
    sq = oracle_tensor_scale(q)
    if dual:                                             # Q1 + Q2
        c1, s1, c2, s2, t = OQ.nvfp4_dual_quantize(f32(q), tensor_scale=sq)
        qh = OQ.nvfp4_dequantize(c1, s1, t) + OQ.nvfp4_dequantize(c2, s2, t)
    else:
        qc, qs, qt = OQ.nvfp4_quantize(f32(q), tensor_scale=sq)
        qh = OQ.nvfp4_dequantize(qc, qs, qt)
    g = hq // hkv
    out = np.zeros((S, hq, d))
    lse = np.zeros((S, hq))
    for s, (k, v) in enumerate(seqs):
        kc, ks, vc, vs = OP.quantize_sequence(f32(k), f32(v), KTS)
        kh = OQ.nvfp4_dequantize(kc, ks, np.float32(KTS))
        vh = OQ.mxfp8_dequantize_v(vc, vs, lens[s])
        for h in range(hkv):
            if exact:                                  # unquantized P, no tiling
                o = OA.exact_attention(qh[s, h * g:(h + 1) * g], kh[h, :lens[s]], vh[h, :lens[s]],
                                       False, scale)
                l = np.zeros(g)
            else:
                o, l = OA.decode_rows(qh[s, h * g:(h + 1) * g], kh[h], vh[h], lens[s], scale, split,
                                      p_underflow_aware=ua)
            out[s, h * g:(h + 1) * g] = o
            lse[s, h * g:(h + 1) * g] = l
    return out, lse


@pytest.mark.parametrize("lens,hq,hkv,split", [([1, 200, 1000, 64, 129], 8, 2, 256),
                                                ([5000, 333], 32, 8, 1024),
                                                ([777], 16, 1, 128),
                                                # g = 8, 1, 3, 6: every softmax instance and
                                                # partial groups of four query columns
                                                ([300, 4100], 16, 2, 512),
                                                ([64, 513], 4, 4, 128),
                                                ([900], 6, 2, 256),
                                                ([130, 700], 12, 2, 256)])
def test_decode_parity(lens, hq, hkv, split):
    d = 128
    cache, table, seqs = _build(lens, hkv, d, seed=sum(lens))
    g = torch.Generator().manual_seed(11)
    q = torch.randn(len(lens), hq, d, generator=g).to(torch.bfloat16)
    q4 = api.quantize_nvfp4(q.to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out, lse = api.attn_qk4v8_decode_paged(q4, cache, table.to(DEV), ctx, max(lens), split,
                                           want_lse=True, out_dtype=torch.float32)
    want, wlse = _oracle_decode(q, seqs, lens, hq, hkv, split, 1 / math.sqrt(d))
    assert_attention_close(f32(out), want, "decode")
    assert np.max(np.abs(lse.cpu().numpy() - wlse)) < 1e-3
    assert api.check_status() == 0


def test_one_split_per_sequence_is_the_one_pass_method():
    """With split_tokens at least the longest context (16384, the largest split the kernel
    takes), every sequence is a single split and the kernel computes the sequential method of
    the BitDecoding-FP4 summary (one running max over the whole cache): parity at the bar
    against the oracle's decode without splits, at 1, 333, 5000 and 16384 tokens."""
    lens, hq, hkv, d = [16384, 5000, 333, 1], 32, 8, 128
    cache, table, seqs = _build(lens, hkv, d, seed=41)
    g = torch.Generator().manual_seed(43)
    q = torch.randn(len(lens), hq, d, generator=g).to(torch.bfloat16)
    q4 = api.quantize_nvfp4(q.to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out, lse = api.attn_qk4v8_decode_paged(q4, cache, table.to(DEV), ctx, max(lens), 16384,
                                           want_lse=True, out_dtype=torch.float32)
    want, wlse = _oracle_decode(q, seqs, lens, hq, hkv, 0, 1 / math.sqrt(d))
    assert_attention_close(f32(out), want, "decode, one split per sequence vs one pass")
    assert np.max(np.abs(lse.cpu().numpy() - wlse)) < 1e-3
    assert api.check_status() == 0


def test_page_permutation_is_bit_invariant():
    lens = [900, 300]
    c1, t1, seqs = _build(lens, 2, 128, seed=5, shuffle=False)
    c2, t2, _ = _build(lens, 2, 128, seed=5, shuffle=True)    # same data, other pages
    q = torch.randn(2, 8, 128, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    q4 = api.quantize_nvfp4(q.to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    o1 = api.attn_qk4v8_decode_paged(q4, c1, t1.to(DEV), ctx, 900, 256)
    o2 = api.attn_qk4v8_decode_paged(q4, c2, t2.to(DEV), ctx, 900, 256)
    assert torch.equal(o1, o2)


@pytest.mark.status_checked
def test_bad_page_id_reports_bounds_error():
    lens = [300]
    cache, table, _ = _build(lens, 2, 128, seed=9)
    table[0, 2] = 10_000                                    # past num_pages
    q4 = api.quantize_nvfp4(torch.randn(1, 8, 128, dtype=torch.bfloat16, device=DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    api.attn_qk4v8_decode_paged(q4, cache, table.to(DEV), ctx, 300, 128)
    assert api.check_status() == 5                          # QK4V8_ERR_BOUNDS
    assert api.check_status() == 0                          # cleared


@pytest.fixture(scope="module")
def paged_workload():
    """The 64-sequence workload (lengths U[8192, 32768], 32/8 heads, shuffled pages) decoded
    once at the benchmark's split of 4096 tokens, fp32 output; the oracle on the shortest, the
    longest and two seeded sequences (all heads) with that split, in one pass (split 0), and
    exact attention on the same quantized operands."""
    lay = workloads.make_decode_layout()
    cfg = lay.cfg
    cache = paged.empty_cache(lay.num_pages, cfg["Hkv"], cfg["d"], KTS, DEV)
    seqs = {}
    lens = lay.lens.tolist()
    pick = {int(np.argmin(lens)), int(np.argmax(lens)), 7, 40}
    for s in range(cfg["S"]):
        k, v = workloads.make_decode_sequence(lay, s)
        n_pages = (lens[s] + 63) // 64
        paged.write_sequence(cache, k.to(DEV), v.to(DEV), lay.page_table[s, :n_pages])
        if s in pick:
            seqs[s] = (k, v)
    q = workloads.make_decode_query(lay)
    q4 = api.quantize_nvfp4(q.to(DEV))
    split = 4096
    out = api.attn_qk4v8_decode_paged(q4, cache, lay.page_table.to(DEV), lay.lens.to(DEV),
                                      max(lens), split, out_dtype=torch.float32)
    assert api.check_status() == 0
    sq = oracle_tensor_scale(q)
    qc, qs, qt = OQ.nvfp4_quantize(f32(q), tensor_scale=sq)
    qh = OQ.nvfp4_dequantize(qc, qs, qt)
    g = cfg["Hq"] // cfg["Hkv"]
    r = {"gpu": [], "split": [], "one_pass": [], "exact": []}
    for s, (k, v) in sorted(seqs.items()):
        kc, ks, vc, vs = OP.quantize_sequence(f32(k), f32(v), KTS)
        kh = OQ.nvfp4_dequantize(kc, ks, np.float32(KTS))
        vh = OQ.mxfp8_dequantize_v(vc, vs, lens[s])
        for h in range(cfg["Hkv"]):
            qq = qh[s, h * g:(h + 1) * g]
            r["split"].append(OA.decode_rows(qq, kh[h], vh[h], lens[s], 1 / math.sqrt(128), split)[0])
            r["one_pass"].append(OA.decode_rows(qq, kh[h], vh[h], lens[s], 1 / math.sqrt(128), 0)[0])
            r["exact"].append(OA.exact_attention(qq, kh[h, :lens[s]], vh[h, :lens[s]], False,
                                                 1 / math.sqrt(128)))
            r["gpu"].append(f32(out[s, h * g:(h + 1) * g]))
    return {k_: np.concatenate(v_) for k_, v_ in r.items()}


def test_paged_workload_sampled_sequences(paged_workload):
    """Parity with the oracle's split-K decode at the kernel's split (4096 tokens)."""
    r = paged_workload
    assert_attention_close(r["gpu"], r["split"], "paged decode workload")


@pytest.mark.xfail(strict=True, reason="split-K reading: each 4096-token split encodes P against "
                   "its own running max, which moves O by E4M3-rounding-level noise (oracle vs "
                   "oracle: 9.3e-2 max, 6.5e-3 mean x rms) -- above the bar against the one-pass method")
def test_split_decode_against_one_pass_method(paged_workload):
    """The benchmark's split-K decode against the sequential one-pass method at the parity
    bar. It does not meet it, by the reading of split-K decode, not by a kernel error: the
    oracle's own split and one-pass decodes differ by the same amount."""
    r = paged_workload
    assert_attention_close(r["gpu"], r["one_pass"], "split 4096 vs one pass")


def test_split_decode_is_no_less_accurate_than_one_pass(paged_workload):
    """The split reading costs no accuracy: against exact attention on the same quantized
    operands, the GPU's split-K decode is at least as close as the one-pass method (measured
    on the oracle: 6.9e-3 against 8.0e-3 mean x rms; the smaller per-split maxima put the
    encoded P values higher in the E4M3 range)."""
    r = paged_workload
    rms = float(np.sqrt(np.mean(r["exact"] ** 2)))
    e_gpu = np.abs(r["gpu"] - r["exact"])
    e_one = np.abs(r["one_pass"] - r["exact"])
    assert e_gpu.mean() <= 1.05 * e_one.mean(), (e_gpu.mean() / rms, e_one.mean() / rms)
    assert e_gpu.max() <= 1.10 * e_one.max(), (e_gpu.max() / rms, e_one.max() / rms)


def test_decode_underflow_aware_parity_and_quality():
    """Rows where one key sits about 14 nats above all others, so every other p~ is below
    2^-10 / 448 and the fixed P scale rounds all of them to zero although together they carry
    a visible share of the weight: with underflow-aware scaling the kernel matches the oracle's
    underflow-aware decode and is several times closer to exact attention than with the fixed
    scale (measured: 2.3e-3 against 2.9e-4 max abs error)."""
    lens, hq, hkv, d, split = [3000, 1700], 8, 2, 128, 1024
    g = torch.Generator().manual_seed(21)
    pages_per = [(n + 63) // 64 for n in lens]
    table = torch.full((len(lens), max(pages_per)), -1, dtype=torch.int32)
    perm = torch.randperm(sum(pages_per), generator=g).int()
    cache = paged.empty_cache(sum(pages_per), hkv, d, KTS, DEV)
    seqs, off = [], 0
    for s, n in enumerate(lens):
        table[s, :pages_per[s]] = perm[off:off + pages_per[s]]
        off += pages_per[s]
        k = torch.full((n, hkv, d), 0.5) + 0.01 * torch.randn(n, hkv, d, generator=g)
        k[n // 3] = 1.75                                   # the top key of every head
        k, v = k.to(torch.bfloat16), (torch.randn(n, hkv, d, generator=g) + 2.0).to(torch.bfloat16)
        seqs.append((k, v))
        paged.write_sequence(cache, k.to(DEV), v.to(DEV), table[s, :pages_per[s]])
    q = torch.ones(len(lens), hq, d).to(torch.bfloat16)
    q4 = api.quantize_nvfp4(q.to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    scale = 1 / math.sqrt(d)
    run = lambda ua: f32(api.attn_qk4v8_decode_paged(q4, cache, table.to(DEV), ctx, max(lens), split,
                                                      out_dtype=torch.float32, underflow_aware=ua))
    out_ua, out_fix = run(True), run(False)
    assert api.check_status() == 0
    want_ua, _ = _oracle_decode(q, seqs, lens, hq, hkv, split, scale, ua=True)
    assert_attention_close(out_ua, want_ua, "decode underflow-aware")
    exact, _ = _oracle_decode(q, seqs, lens, hq, hkv, split, scale, exact=True)
    err_fix = np.abs(out_fix - exact).max()
    err_ua = np.abs(out_ua - exact).max()
    assert err_fix > 1e-3 and err_fix > 5 * err_ua, (err_fix, err_ua)


@pytest.mark.parametrize("ua", [False, True])
def test_decode_dual_q_parity(ua):
    """Dual-residual Q (and with underflow-aware P): the kernel matches the oracle's decode
    with Q1 + Q2."""
    lens, hq, hkv, d, split = [5000, 333, 1], 32, 8, 128, 1024
    cache, table, seqs = _build(lens, hkv, d, seed=77)
    g = torch.Generator().manual_seed(12)
    q = torch.randn(len(lens), hq, d, generator=g)
    q[..., :4] *= 8
    q = q.to(torch.bfloat16)
    q1, q2 = api.quantize_nvfp4_dual(q.to(DEV))
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    out = api.attn_qk4v8_decode_paged(q1, cache, table.to(DEV), ctx, max(lens), split,
                                      out_dtype=torch.float32, underflow_aware=ua, q2=q2)
    assert api.check_status() == 0
    want, _ = _oracle_decode(q, seqs, lens, hq, hkv, split, 1 / math.sqrt(d), ua=ua, dual=True)
    assert_attention_close(f32(out), want, "decode dual Q")


def test_decode_plan_matches_the_call():
    """DecodePlan (fixed buffers checked once, only the query changes per step) gives the same
    bytes as attn_qk4v8_decode_paged on two steps in a row, and rejects a query of another
    shape."""
    lens, hq, hkv, d, split = [700, 64, 1500], 8, 2, 128, 512
    cache, table, _ = _build(lens, hkv, d, seed=31)
    ctx = torch.tensor(lens, dtype=torch.int32, device=DEV)
    table = table.to(DEV)
    plan = api.DecodePlan(cache, table, ctx, max(lens), split, len(lens), hq, want_lse=True)
    g = torch.Generator().manual_seed(3)
    for _ in range(2):
        q4 = api.quantize_nvfp4(torch.randn(len(lens), hq, d, generator=g).to(torch.bfloat16).to(DEV))
        out, lse = plan.run(q4)
        ref, rlse = api.attn_qk4v8_decode_paged(q4, cache, table, ctx, max(lens), split, want_lse=True)
        assert torch.equal(out, ref) and torch.equal(lse, rlse)
    bad = api.quantize_nvfp4(torch.randn(len(lens), hq // 2, d).to(torch.bfloat16).to(DEV))
    with pytest.raises(ValueError):
        plan.run(bad)
