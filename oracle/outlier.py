"""Oracle — outlier-aware key quantization (TEST INFRASTRUCTURE ONLY; see oracle/formats.py).

sns.style BitDecoding-FP4 summary, third algorithm item: key tensors carry outlier channels
that stretch the range a scale must cover; static smoothing and a Hadamard rotation first
spread the outliers' energy, then a scale search picks a better scale per group. The page gives
no formulas; the readings:

* Static smoothing: one positive factor lam_c per channel, fixed in advance (calibration);
  keys are divided by it and queries multiplied by it, so every logit is unchanged:
  k'_c = fl32(k_c / lam_c), q'_c = fl32(q_c * lam_c).
* Rotation: x -> (x H) 2^-e with H the 128 x 128 Sylvester Walsh-Hadamard matrix (entries
  +-1, H H^T = 128 I), as seven butterfly stages in float32: stage s = 0..6 replaces each pair
  (i, i + 2^s), bit s of i clear, by (a + b, a - b). Queries take e = 3 and keys e = 4, so that
  (q H 2^-3)(k H 2^-4)^T = q k^T exactly. The result is rounded once to the stored 16-bit type.
* Scale search (keys): per 16-element block the E4M3 scale codes c0, c0 - 1, c0 - 2, c0 + 1
  (c0 the usual E4M3(fl32(fl32(amax_b / 6) / s_t)); codes outside 1..126 skipped) each encode
  the block (den = fl32(decode(c) s_t), codes E2M1(fl32(x / den))); the block error is
  err = sum over i = 0..15 in order of fl32(d_i * d_i), d_i = fl32(x_i - fl32(value_i * den)),
  accumulated with float32 adds; the smallest error wins, ties to the earlier candidate.
"""
from __future__ import annotations

import numpy as np

from .formats import e2m1_decode, e2m1_encode, e4m3_decode, e4m3_encode, fp16_round
from .quant import NVFP4_BLOCK, nvfp4_tensor_scale

F32 = np.float32


def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 -> nearest bfloat16 (ties to even), returned as float32 (finite inputs)."""
    u = np.asarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(F32)


def hadamard_rows(x: np.ndarray) -> np.ndarray:
    """x H along the last axis (length 128), by the butterfly stages, in float32."""
    y = np.array(x, dtype=F32, copy=True)
    n = y.shape[-1]
    assert n == 128
    for s in range(7):
        h = 1 << s
        v = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a, b = v[..., 0, :].copy(), v[..., 1, :].copy()
        v[..., 0, :] = a + b
        v[..., 1, :] = a - b
    return y


def smooth_rotate(x: np.ndarray, lam: np.ndarray | None, role: str, dtype: str) -> np.ndarray:
    """Smoothing (role 'q' multiplies by lam, 'k' divides), rotation, 2^-3 (q) or 2^-4 (k), and
    one rounding to ``dtype`` ('bf16' or 'fp16'). Returns the stored values as float32."""
    y = np.asarray(x, dtype=F32)
    if lam is not None:
        lam = np.asarray(lam, dtype=F32)
        y = (y * lam) if role == "q" else (y / lam)
        y = y.astype(F32)
    y = hadamard_rows(y) * F32(2.0 ** (-3 if role == "q" else -4))
    return bf16_round(y) if dtype == "bf16" else fp16_round(y).astype(F32)


def nvfp4_quantize_searched(x: np.ndarray, tensor_scale: float | None = None):
    """NVFP4 with a per-block scale search (module docstring). Returns (packed, scales, s_t)."""
    x = np.asarray(x, dtype=F32)
    cols = x.shape[-1]
    s_t = nvfp4_tensor_scale(x) if tensor_scale is None else F32(tensor_scale)
    blocks = x.reshape(-1, NVFP4_BLOCK)
    amax_b = np.max(np.abs(blocks), axis=-1)
    c0 = e4m3_encode(((amax_b / F32(6.0)).astype(F32) / s_t).astype(F32)).astype(np.int64)
    best_code = c0.copy()
    best_err = np.full(blocks.shape[0], np.inf, dtype=np.float64)
    best_e2 = np.zeros(blocks.shape, dtype=np.uint8)
    for off in (0, -1, -2, 1):
        c = c0 + off
        ok = (c >= 1) & (c <= 126) & (c0 >= 1)
        cc = np.clip(c, 0, 126)
        den = (e4m3_decode(cc.astype(np.uint8)).astype(F32) * s_t).astype(F32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = (blocks / den[:, None]).astype(F32)
        e2 = e2m1_encode(q)
        vals = e2m1_decode(e2).astype(F32)
        err = np.zeros(blocks.shape[0], dtype=F32)
        for i in range(NVFP4_BLOCK):
            d = (blocks[:, i] - (vals[:, i] * den).astype(F32)).astype(F32)
            err = (err + (d * d).astype(F32)).astype(F32)
        take = ok & (err.astype(np.float64) < best_err)
        best_err = np.where(take, err, best_err)
        best_code = np.where(take, c, best_code)
        best_e2 = np.where(take[:, None], e2, best_e2)
    zero = c0 == 0                                          # decode(s_b) = 0: all codes 0
    best_e2[zero] = 0
    best_code[zero] = 0
    codes = best_e2.reshape(x.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, best_code.reshape(x.shape[:-1] + (cols // NVFP4_BLOCK,)).astype(np.uint8), s_t
