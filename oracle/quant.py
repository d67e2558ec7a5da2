"""Oracle — NVFP4 and MXFP8 quantizers (TEST INFRASTRUCTURE ONLY; see oracle/formats.py).

NVFP4 (Q and K). Structure from the tqpw.cn "块缩放数值格式" article §2.2: E2M1 elements,
one E4M3 scale per 16 consecutive elements, one FP32 scale per tensor (the article describes
a two-level scaling: a tensor-wide FP32 factor above small 16-element blocks). The article's own listing has the wrong
arithmetic (raw amax as global scale, no division by 6, an integer grid); the reading used
here is the plainest one that keeps every block scale representable in E4M3:

    amax_t = max |x| over the tensor passed in                (exact)
    s_t    = fl32(amax_t / 2688)        (2688 = 6 * 448);  amax_t == 0  ->  s_t = 1
    per block of 16 along the last axis:
        s_b    = E4M3( fl32( fl32(amax_b / 6) / s_t ) )      (two FP32 divides, in order)
        den    = fl32( decode(s_b) * s_t )
        code_i = E2M1( fl32(x_i / den) );   decode(s_b) == 0  ->  every code is 0x0
    x_hat_i = decode(code_i) * decode(s_b) * s_t             (float64)

All FP32 steps are single IEEE operations rounded to nearest (numpy float32 arithmetic);
subnormals are kept. A caller-supplied tensor scale replaces s_t (used for a KV cache whose
scale is fixed in advance). Packing: element 2i in the low nibble, 2i+1 in the high nibble.

MXFP8 (V). The tqpw.cn article §2.1 and the zdszero primer (MXFP8 section: an E8M0 scale for
each 1x32 block) fix E4M3 elements with one E8M0 scale per 32 elements. The shared-exponent rule is not
on the pages; the OCP MX rule is used: e = floor(log2 amax) - 8 (8 is the exponent of E4M3's
largest normal, 448 = 1.75 * 2^8), clamped to [-127, 127]; scale code e + 127; elements
E4M3(v / 2^e); an all-zero group gets scale code 127 and zero codes. Groups run along the
token axis (the PV contraction), per channel; a group cut short by the end of the sequence
uses the tokens present, and padding codes are 0.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode

NVFP4_BLOCK = 16
MXFP8_BLOCK = 32
F32 = np.float32


def nvfp4_tensor_scale(x: np.ndarray) -> np.float32:
    """s_t = fl32(amax / 2688), or 1 for an all-zero tensor."""
    amax = F32(np.max(np.abs(np.asarray(x, dtype=F32)))) if np.size(x) else F32(0)
    if amax == 0:
        return F32(1.0)
    return F32(amax / F32(2688.0))


def nvfp4_quantize(x: np.ndarray, tensor_scale: float | None = None):
    """Quantize ``x`` (..., cols), cols % 16 == 0, to NVFP4.

    Returns (codes uint8 (..., cols//2) packed, scales uint8 (..., cols//16) E4M3 codes,
    s_t float32).
    """
    x = np.asarray(x, dtype=F32)
    cols = x.shape[-1]
    assert cols % NVFP4_BLOCK == 0
    s_t = nvfp4_tensor_scale(x) if tensor_scale is None else F32(tensor_scale)
    blocks = x.reshape(x.shape[:-1] + (cols // NVFP4_BLOCK, NVFP4_BLOCK))
    amax_b = np.max(np.abs(blocks), axis=-1)                       # exact, float32
    sb_f32 = (amax_b / F32(6.0)).astype(F32) / s_t                 # two IEEE divides
    sb_code = e4m3_encode(sb_f32.astype(F32))
    sb_val = e4m3_decode(sb_code).astype(F32)                      # exact in float32
    den = (sb_val * s_t).astype(F32)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (blocks / den[..., None]).astype(F32)
    codes = e2m1_encode(ratio)
    codes = np.where((sb_val == 0)[..., None], np.uint8(0), codes).astype(np.uint8)
    codes = codes.reshape(x.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, sb_code.astype(np.uint8), s_t


def nvfp4_unpack(packed: np.ndarray) -> np.ndarray:
    """(..., cols//2) packed bytes -> (..., cols) 4-bit codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def nvfp4_dequantize(packed: np.ndarray, scales: np.ndarray, s_t: float) -> np.ndarray:
    """x_hat = decode(code) * decode(s_b) * s_t, in float64."""
    codes = nvfp4_unpack(packed)
    vals = e2m1_decode(codes)
    cols = vals.shape[-1]
    sb = e4m3_decode(scales)
    vals = vals.reshape(vals.shape[:-1] + (cols // NVFP4_BLOCK, NVFP4_BLOCK))
    return (vals * sb[..., None] * np.float64(s_t)).reshape(codes.shape)


def nvfp4_residual(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, s_t) -> np.ndarray:
    """The part of ``x`` its NVFP4 encoding (packed, scales, s_t) misses, in FP32 steps:
    den = fl32(decode(s_b) * s_t), d_i = fl32(decode(code_i) * den), r_i = fl32(x_i - d_i)."""
    x = np.asarray(x, dtype=F32)
    cols = x.shape[-1]
    vals = e2m1_decode(nvfp4_unpack(packed)).astype(F32)            # exact small values
    vals = vals.reshape(vals.shape[:-1] + (cols // NVFP4_BLOCK, NVFP4_BLOCK))
    den = (e4m3_decode(scales).astype(F32) * F32(s_t)).astype(F32)
    d = (vals * den[..., None]).astype(F32)
    blocks = x.reshape(vals.shape)
    return (blocks - d).astype(F32).reshape(x.shape)


def nvfp4_dual_quantize(x: np.ndarray, tensor_scale: float | None = None):
    """Dual-residual NVFP4 (sns.style BitDecoding-FP4 summary, first algorithm item: the query
    is split into two FP4 tensors, the second carrying what the first leaves over). Reading:
    Q1 = NVFP4(x); Q2 = NVFP4(x - x_hat1) with the same tensor scale s_t, so that Q1 K^T and
    Q2 K^T share one accumulator. Returns (codes1, scales1, codes2, scales2, s_t)."""
    c1, s1, s_t = nvfp4_quantize(x, tensor_scale)
    c2, s2, _ = nvfp4_quantize(nvfp4_residual(x, c1, s1, s_t), tensor_scale=s_t)
    return c1, s1, c2, s2, s_t


def mxfp8_round_up_tokens(n: int) -> int:
    """Token extent of the stored V codes: whole 128-token tiles."""
    return (n + 127) // 128 * 128


def mxfp8_group_exponent(amax: np.ndarray) -> np.ndarray:
    """e = floor(log2 amax) - 8, clamped to [-127, 127]; amax == 0 -> 0 (code 127)."""
    amax = np.asarray(amax, dtype=np.float64)
    e = np.zeros(amax.shape, dtype=np.int64)
    nz = amax > 0
    _, ex = np.frexp(amax[nz])
    e[nz] = (ex - 1) - 8
    return np.clip(e, -127, 127)


def mxfp8_quantize_v(v: np.ndarray):
    """Quantize V laid out (..., N, d) to MXFP8 along the token axis.

    Returns (codes uint8 (..., d, N_pad) token-contiguous, scales uint8 (..., d, N_pad//32)
    E8M0 codes), N_pad = N rounded up to a multiple of 128.
    """
    v = np.asarray(v, dtype=F32)
    n, d = v.shape[-2], v.shape[-1]
    n_pad = mxfp8_round_up_tokens(n)
    vt = np.zeros(v.shape[:-2] + (d, n_pad), dtype=np.float64)
    vt[..., :n] = np.swapaxes(v, -1, -2)
    groups = vt.reshape(vt.shape[:-1] + (n_pad // MXFP8_BLOCK, MXFP8_BLOCK))
    amax = np.max(np.abs(groups), axis=-1)
    e = mxfp8_group_exponent(amax)
    scaled = groups / np.ldexp(1.0, e)[..., None]                  # exact power-of-two divide
    codes = e4m3_encode(scaled).reshape(vt.shape)
    codes[..., n:] = 0
    return codes.astype(np.uint8), (e + 127).astype(np.uint8)


def mxfp8_dequantize_v(codes: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    """Inverse layout of ``mxfp8_quantize_v``: returns v_hat (..., n, d) float64."""
    vals = e4m3_decode(codes)
    d, n_pad = vals.shape[-2], vals.shape[-1]
    groups = vals.reshape(vals.shape[:-1] + (n_pad // MXFP8_BLOCK, MXFP8_BLOCK))
    deq = (groups * np.ldexp(1.0, scales.astype(np.int64) - 127)[..., None]).reshape(vals.shape)
    return np.swapaxes(deq[..., :n], -1, -2)
