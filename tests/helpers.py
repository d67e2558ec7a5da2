"""Shared helpers of the GPU parity tests: run the oracle on the same seeded inputs the CUDA
path gets, and the attention tolerance of the problem statement."""
import math

import numpy as np
import torch

from oracle import attention as OA
from oracle import formats as OF
from oracle import quant as OQ
from oracle import tilescore as OT

#: Attention parity bar: max |O_gpu - O_oracle| <= 2e-2 rms(O_oracle) and mean <= 2e-3 rms.
MAX_TOL = 2e-2
MEAN_TOL = 2e-3


def f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def attention_error(out_gpu: np.ndarray, out_oracle: np.ndarray):
    rms = float(np.sqrt(np.mean(out_oracle.astype(np.float64) ** 2)))
    d = np.abs(out_gpu.astype(np.float64) - out_oracle)
    return float(d.max()) / rms, float(d.mean()) / rms


def assert_attention_close(out_gpu, out_oracle, what=""):
    mx, mean = attention_error(out_gpu, out_oracle)
    assert np.all(np.isfinite(out_gpu)), what
    assert mx <= MAX_TOL and mean <= MEAN_TOL, f"{what}: max {mx:.3e} mean {mean:.3e} (x rms)"
    return mx, mean


def oracle_output(out_oracle, dtype):
    """The oracle's O as the method defines a 16-bit output: the float64 O / l rounded once to
    the output dtype (fp32 outputs are compared with the float64 values)."""
    if dtype == torch.bfloat16:
        return OF.bf16_round(out_oracle)
    if dtype == torch.float16:
        return OF.fp16_round(out_oracle)
    return out_oracle


def round_to_output(x, dtype):
    """float values rounded once to a 16-bit output dtype (float64 in, float64 out)."""
    return OF.bf16_round(x) if dtype == torch.bfloat16 else OF.fp16_round(x)


def assert_rounded_output_close(out16, out32, out_oracle, dtype, what=""):
    """Parity of a 16-bit output, with no allowance added to the bar:

    * the 16-bit output is the same kernel's fp32 output rounded once to that dtype, bit for
      bit (the fp32 output itself is held to the plain bar by the caller);
    * against the oracle's O rounded once to that dtype, the mean error is within the plain
      bar, and every element over the plain max bar is exactly one unit in the last place of
      the output format away (the two unrounded values straddle a rounding boundary; one bf16
      unit at |O| > 2.56 rms is already more than 2e-2 rms, so no kernel could meet the max bar
      there), on at most one element in 10^4.
    """
    ref16 = round_to_output(out_oracle, dtype)
    assert np.array_equal(out16, round_to_output(out32.astype(np.float64), dtype)), \
        f"{what}: the 16-bit output is not the fp32 output rounded once"
    rms = float(np.sqrt(np.mean(out_oracle.astype(np.float64) ** 2)))
    d = np.abs(out16.astype(np.float64) - ref16)
    assert np.all(np.isfinite(out16)), what
    assert d.mean() <= MEAN_TOL * rms, f"{what}: mean {d.mean() / rms:.3e} (x rms)"
    over = d > MAX_TOL * rms
    if over.any():
        mant = {torch.bfloat16: 8, torch.float16: 11}[dtype]
        mag = np.maximum(np.abs(out16[over]).astype(np.float64), np.abs(ref16[over]))
        ulp = np.ldexp(1.0, np.frexp(mag)[1] - mant)           # one unit at the larger one
        lower = np.ldexp(1.0, np.frexp(np.minimum(np.abs(out16[over]), np.abs(ref16[over])))[1] - mant)
        assert np.all((d[over] == ulp) | (d[over] == lower)), f"{what}: an element off by more than one unit"
        assert over.sum() <= max(1, d.size // 10000), f"{what}: {over.sum()} elements one unit apart"


def oracle_tensor_scale(x: torch.Tensor) -> np.float32:
    """The NVFP4 tensor scale of a whole (possibly large) tensor, computed chunk-wise."""
    amax = np.float32(0)
    flat = x.reshape(-1)
    for i in range(0, flat.numel(), 1 << 26):
        amax = max(amax, np.float32(flat[i:i + (1 << 26)].float().abs().max().item()))
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2688.0))


def oracle_nvfp4(x: torch.Tensor, s_t=None):
    """Oracle NVFP4 of a CPU tensor (..., D) with the tensor scale s_t (computed if None)."""
    return OQ.nvfp4_quantize(f32(x), tensor_scale=s_t)


def oracle_dequant_q(x: torch.Tensor, s_t=None):
    c, s, t = oracle_nvfp4(x, s_t)
    return OQ.nvfp4_dequantize(c, s, t), (c, s, t)


def oracle_prefill_rows(q, k, v, hq, rows, causal, scale, hkv_of=None, fp16_select=None):
    """Oracle attention for query head ``hq`` (batch 0) at query ``rows`` of bf16/fp16 CPU
    tensors q [B, Hq, N, D], k/v [B, Hkv, N, D]; quantization with whole-tensor scales."""
    B, Hq, N, D = q.shape
    Hkv = k.shape[1]
    hk = hq // (Hq // Hkv)
    sq = oracle_tensor_scale(q)
    sk = oracle_tensor_scale(k)
    qh, _ = oracle_dequant_q(q[0, hq, rows], sq)
    kh, _ = oracle_dequant_q(k[0, hk], sk)
    vc, vs = OQ.mxfp8_quantize_v(f32(v[0, hk]))
    vh = OQ.mxfp8_dequantize_v(vc, vs, v.shape[2])
    kw = {}
    if fp16_select is not None:
        # FP16 tiles: Q and K as given (16-bit values, multiplied exactly), V rounded to fp16
        kw = dict(fp16_select=fp16_select, q16=f32(q[0, hq, rows]).astype(np.float64),
                  k16=f32(k[0, hk]).astype(np.float64), v16=OF.fp16_round(f32(v[0, hk])))
    m, l, o = OA.attention_rows(qh, np.asarray(rows), kh, vh, causal, scale, **kw)
    return OA.finish(m, l, o)
