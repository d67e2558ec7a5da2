"""GPU parity of the QK4V8 prefill attention against the oracle (max |dO| <= 2e-2 rms and
mean <= 2e-3 rms), full outputs on the small workloads and ragged shapes, sampled rows on the
long-context workload, plus exact invariants on the GPU path itself."""
import math

import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, workloads
from oracle import attention as OA
from oracle import quant as OQ
from helpers import (assert_attention_close, assert_rounded_output_close, f32,
                     oracle_prefill_rows, oracle_tensor_scale)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(q, k, v, causal, scale=None, frac_bp=0, out_dtype=torch.float32, ua=False, dual=False):
    return api.qk4v8_attention(q.to(DEV), k.to(DEV), v.to(DEV), causal, scale,
                               fp16_frac_bp=frac_bp, out_dtype=out_dtype, underflow_aware=ua,
                               dual_q=dual)


def _full_oracle(q, k, v, causal, scale, ua=False, exact=False, dual=False, q_exact=False):
    B, Hq, N, D = q.shape
    out = np.zeros((B, Hq, q.shape[2], D))
    Hkv = k.shape[1]
    sq, sk = oracle_tensor_scale(q), oracle_tensor_scale(k)
    for b in range(B):
        for hk in range(Hkv):
            kh = OQ.nvfp4_dequantize(*OQ.nvfp4_quantize(f32(k[b, hk]), tensor_scale=sk))
            vc, vs = OQ.mxfp8_quantize_v(f32(v[b, hk]))
            vh = OQ.mxfp8_dequantize_v(vc, vs, v.shape[2])
            for hq in range(hk * (Hq // Hkv), (hk + 1) * (Hq // Hkv)):
                if q_exact:                            # the unquantized query
                    qh = f32(q[b, hq]).astype(np.float64)
                elif dual:                             # Q1 + Q2
                    c1, s1, c2, s2, t = OQ.nvfp4_dual_quantize(f32(q[b, hq]), tensor_scale=sq)
                    qh = OQ.nvfp4_dequantize(c1, s1, t) + OQ.nvfp4_dequantize(c2, s2, t)
                else:
                    qh = OQ.nvfp4_dequantize(*OQ.nvfp4_quantize(f32(q[b, hq]), tensor_scale=sq))
                if exact:
                    out[b, hq] = OA.exact_attention(qh, kh, vh, causal, scale)
                else:
                    out[b, hq] = OA.attention_head(qh, kh, vh, causal, scale,
                                                   p_underflow_aware=ua)[0]
    return out


@pytest.mark.parametrize("name", ["tiny_prefill", "prefill_h16_n4096"])
def test_workload_full_parity(name):
    w = workloads.make_prefill(name)
    D = w.cfg["d"]
    scale = 1 / math.sqrt(D)
    out = _run(w.q, w.k, w.v, w.cfg["causal"], scale)
    ref = _full_oracle(w.q, w.k, w.v, w.cfg["causal"], scale)
    assert_attention_close(f32(out), ref, name)
    out16 = _run(w.q, w.k, w.v, w.cfg["causal"], scale, out_dtype=w.q.dtype)
    assert out16.dtype == w.q.dtype
    assert_rounded_output_close(f32(out16), f32(out), ref, w.q.dtype, name + " 16-bit output")


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,D,causal", [
    (1, 4, 2, 300, 300, 128, True),      # GQA, ragged tail
    (2, 2, 1, 1000, 1000, 64, False),    # batch 2, non-causal, D = 64
    (1, 2, 2, 200, 700, 128, False),     # Nq != Nk
    (1, 1, 1, 1, 1, 128, True),          # one token
    (1, 3, 3, 129, 129, 64, True),
    (1, 3, 1, 300, 300, 128, True),      # odd GQA ratio: consecutive query tiles paired, the last alone
    (2, 2, 2, 520, 520, 64, True),       # five query tiles a head: pairs and a lone last tile
    (1, 2, 2, 390, 390, 128, False),     # the same without the causal mask
])
def test_ragged_shapes(B, Hq, Hkv, Nq, Nk, D, causal):
    g = torch.Generator().manual_seed(Nq * 7 + Nk)
    q = torch.randn(B, Hq, Nq, D, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, Hkv, Nk, D, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nk, D, generator=g).to(torch.bfloat16)
    out = _run(q, k, v, causal)
    ref = _full_oracle(q, k, v, causal, 1 / math.sqrt(D))
    assert_attention_close(f32(out), ref, "ragged")


def test_long_context_gqa_sampled():
    """32 query / 8 KV heads, 32768 tokens, causal; oracle on 2 heads x 256 seeded rows."""
    w = workloads.make_prefill("prefill_gqa_n32768")
    scale = 1 / math.sqrt(128)
    out = _run(w.q, w.k, w.v, True, scale)
    rng = np.random.default_rng(2)
    heads = sorted(rng.choice(32, size=2, replace=False).tolist())
    got, want = [], []
    for hq in heads:
        rows = np.sort(rng.choice(32768, size=256, replace=False))
        o, _ = oracle_prefill_rows(w.q, w.k, w.v, hq, rows, True, scale)
        want.append(o)
        got.append(f32(out[0, hq, torch.as_tensor(rows, device=DEV)]))
    assert_attention_close(np.concatenate(got), np.concatenate(want), "gqa 32k sampled")


def test_constant_v_gives_constant_output():
    g = torch.Generator().manual_seed(0)
    q = torch.randn(1, 2, 500, 128, generator=g).to(torch.bfloat16)
    k = (torch.randn(1, 2, 500, 128, generator=g) * 3).to(torch.bfloat16)
    v = torch.ones(1, 2, 500, 128, dtype=torch.bfloat16)
    out = _run(q, k, v, True)
    assert torch.all((out - 1.0).abs() <= 2.0 ** -20)


def test_first_causal_row_is_dequantized_v0():
    w = workloads.make_prefill("prefill_h16_n4096")
    out = _run(w.q, w.k, w.v, True)
    vc, vs = OQ.mxfp8_quantize_v(f32(w.v[0, 3]))
    v0 = OQ.mxfp8_dequantize_v(vc, vs, 4096)[0]
    assert np.array_equal(f32(out[0, 3, 0]), v0.astype(np.float32))


def test_lse_matches_oracle():
    g = torch.Generator().manual_seed(3)
    q = torch.randn(1, 2, 256, 128, generator=g).to(torch.bfloat16)
    k = torch.randn(1, 2, 256, 128, generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, 256, 128, generator=g).to(torch.bfloat16)
    q4, k4, v8 = api.quantize_nvfp4(q.to(DEV)), api.quantize_nvfp4(k.to(DEV)), api.quantize_mxfp8_v(v.to(DEV))
    _, lse = api.attn_qk4v8_fwd(q4, k4, v8, True, want_lse=True)
    _, want = oracle_prefill_rows(q, k, v, 1, np.arange(256), True, 1 / math.sqrt(128))
    assert np.max(np.abs(lse[0, 1].cpu().numpy() - want)) < 1e-3


def test_bf16_output_workload_long_rows():
    """A bf16 output (2000 causal rows, g = 2) matches the oracle's O rounded once to bf16."""
    g = torch.Generator().manual_seed(4)
    q = torch.randn(1, 2, 2000, 128, generator=g).to(torch.bfloat16)
    k = (torch.randn(1, 1, 2000, 128, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(1, 1, 2000, 128, generator=g).to(torch.bfloat16)
    out = _run(q, k, v, True, out_dtype=torch.bfloat16)
    out32 = _run(q, k, v, True, out_dtype=torch.float32)
    ref = _full_oracle(q, k, v, True, 1 / math.sqrt(128))
    assert_attention_close(f32(out32), ref, "fp32 output")
    assert_rounded_output_close(f32(out), f32(out32), ref, torch.bfloat16, "bf16 output")


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,D,causal", [
    (1, 4, 2, 700, 700, 128, True),
    (1, 2, 1, 300, 900, 64, False),
])
def test_underflow_aware_parity(B, Hq, Hkv, Nq, Nk, D, causal):
    """Peaky scores (K x 6), so most 32-key blocks take a scale below 1: the underflow-aware
    kernel matches the oracle's underflow-aware attention."""
    g = torch.Generator().manual_seed(Nq + Nk + D)
    q = torch.randn(B, Hq, Nq, D, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, Hkv, Nk, D, generator=g) * 6).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nk, D, generator=g).to(torch.bfloat16)
    out = _run(q, k, v, causal, ua=True)
    ref = _full_oracle(q, k, v, causal, 1 / math.sqrt(D), ua=True)
    assert_attention_close(f32(out), ref, "underflow-aware")


def test_underflow_aware_keeps_the_small_keys():
    """One key about 14 nats above 2047 others: the fixed P scale rounds all of those to zero,
    the underflow-aware one keeps them and is several times closer to exact attention."""
    n, d = 2048, 128
    q = torch.ones(1, 2, n, d).to(torch.bfloat16)
    k = torch.full((1, 1, n, d), 0.5) + 0.01 * torch.randn(1, 1, n, d, generator=torch.Generator().manual_seed(2))
    k[0, 0, 7] = 1.75
    k = k.to(torch.bfloat16)
    v = (torch.randn(1, 1, n, d, generator=torch.Generator().manual_seed(3)) + 2.0).to(torch.bfloat16)
    scale = 1 / math.sqrt(d)
    exact = _full_oracle(q, k, v, False, scale, exact=True)
    err = {ua: np.abs(f32(_run(q, k, v, False, scale, ua=ua)) - exact).max() for ua in (False, True)}
    assert err[False] > 1e-3 and err[False] > 5 * err[True], err


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,D,causal", [
    (1, 4, 2, 700, 700, 128, True),
    (1, 2, 1, 300, 900, 64, False),
])
def test_dual_q_parity_and_quality(B, Hq, Hkv, Nq, Nk, D, causal):
    """Dual-residual Q: the kernel matches the oracle's attention with Q1 + Q2, and it is closer
    than the single-Q kernel to the attention whose query is not quantized at all."""
    g = torch.Generator().manual_seed(Nq * 3 + D)
    q = torch.randn(B, Hq, Nq, D, generator=g)
    q[..., :4] *= 8                                      # outlier channels make Q1 coarse
    q = q.to(torch.bfloat16)
    k = (torch.randn(B, Hkv, Nk, D, generator=g) * 2).to(torch.bfloat16)
    v = torch.randn(B, Hkv, Nk, D, generator=g).to(torch.bfloat16)
    scale = 1 / math.sqrt(D)
    out2 = f32(_run(q, k, v, causal, scale, dual=True))
    assert_attention_close(out2, _full_oracle(q, k, v, causal, scale, dual=True), "dual Q")
    ref = _full_oracle(q, k, v, causal, scale, q_exact=True)
    out1 = f32(_run(q, k, v, causal, scale))
    e1, e2 = np.abs(out1 - ref).mean(), np.abs(out2 - ref).mean()
    assert e2 < e1 / 2, (e1, e2)
