"""Oracle — element formats of the QK4V8 path (TEST INFRASTRUCTURE ONLY).

This package is the slow, plain CPU restatement used to check the CUDA library. Only the
test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it; the library never does, and it imports nothing from the library.

Formats (all decoded in float64, exactly):

* E2M1 ("FP4"): 1 sign, 2 exponent, 1 mantissa bit, exponent bias 1. Magnitudes
  {0, 0.5, 1, 1.5, 2, 3, 4, 6}. Source: zdszero "quantization" primer, floating-point
  format table (row fp4(e2m1)); tqpw.cn "块缩放数值格式" article §2.2 (element-level 4-bit
  FP4 E2M1 in NVFP4).
* E4M3 ("e4m3fn"): 1/4/3 bits, bias 7, subnormals m*2^-9 at exponent 0, S.1111.111 is NaN,
  no infinity, largest finite 448. Source: zdszero primer, format table row fp8(e4m3);
  tqpw.cn article §2.2 (block-level 8-bit E4M3 scale factor).
* E8M0: unsigned 8-bit pure exponent, value 2^(e-127), 0xFF is NaN. Source: tqpw.cn
  article §2.1 (MXFP scale factor is an 8-bit exponent E8M0). The primer's table lists a sign
  bit for e8m0; that row is garbled — E8M0 carries no sign.

Encoders round to nearest, ties to even mantissa, and saturate to the largest finite
magnitude (the "satfinite" reading: no format here has an infinity). The sign of a value is
kept when it rounds to zero (a negative input that rounds to zero encodes as negative zero).
That last point is a reading: the pages are silent on signed zeros.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------------------
# E2M1
# ---------------------------------------------------------------------------------------

#: The eight non-negative E2M1 magnitudes, indexed by the low three code bits (eem).
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)
E2M1_MAX = 6.0


def e2m1_decode_closed_form(code: int) -> float:
    """Decode one E2M1 code from its bit fields (bias 1; exponent 0 is subnormal)."""
    sign = -1.0 if (code >> 3) & 1 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    if e == 0:
        mag = 0.5 * m                      # subnormal: 2^(1-1) * (m/2)
    else:
        mag = 2.0 ** (e - 1) * (1.0 + 0.5 * m)
    return sign * mag


#: Full 16-entry decode table, built from the closed form.
E2M1_TABLE = np.array([e2m1_decode_closed_form(c) for c in range(16)], dtype=np.float64)


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_TABLE[np.asarray(codes, dtype=np.uint8) & 0xF]


# Decision points between neighbouring magnitudes: 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.
_E2M1_MIDPOINTS = 0.5 * (E2M1_MAGNITUDES[:-1] + E2M1_MAGNITUDES[1:])


def e2m1_encode(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even, saturating E2M1 encode of finite values (any float dtype).

    The magnitude code is the number of decision points strictly below |x|; when |x| sits
    exactly on a decision point the two neighbours tie and the even code (mantissa bit 0)
    wins. Anything above 6 saturates to code 7 (6.0).
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    c = np.searchsorted(_E2M1_MIDPOINTS, a, side="left")          # mids strictly below a
    tie = np.zeros(a.shape, dtype=bool)
    inside = c < len(_E2M1_MIDPOINTS)
    tie[inside] = a[inside] == _E2M1_MIDPOINTS[c[inside]]
    c = np.where(tie & (c % 2 == 1), c + 1, c)                     # tie: take the even code
    sign = np.signbit(x).astype(np.int64)
    return ((sign << 3) | c).astype(np.uint8)


# ---------------------------------------------------------------------------------------
# E4M3 (e4m3fn)
# ---------------------------------------------------------------------------------------

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6
E4M3_MANT_BITS = 3


def e4m3_decode_closed_form(code: int) -> float:
    sign = -1.0 if (code >> 7) & 1 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0xF and m == 7:
        return float("nan")
    if e == 0:
        mag = m * 2.0 ** -9                # subnormal: 2^(1-7) * (m/8)
    else:
        mag = 2.0 ** (e - 7) * (1.0 + m / 8.0)
    return sign * mag


E4M3_TABLE = np.array([e4m3_decode_closed_form(c) for c in range(256)], dtype=np.float64)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    return E4M3_TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Value of the round-to-nearest-even, saturating E4M3 conversion, as float64.

    For |x| with binary exponent E = floor(log2|x|) (never below the smallest normal
    exponent -6), the grid spacing is 2^(E-3); |x| / spacing is exact in float64 and
    ``np.rint`` rounds it half-to-even. Results above 448 saturate to 448.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    nz = a > 0
    e = np.zeros(a.shape, dtype=np.int64)
    _, ex = np.frexp(a[nz])                   # a = f * 2^ex, f in [0.5, 1)
    e[nz] = ex - 1
    e = np.maximum(e, E4M3_MIN_NORMAL_EXP)
    q = np.ldexp(1.0, e - E4M3_MANT_BITS)
    r = np.rint(a / q) * q
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even, saturating E4M3 encode of finite values -> uint8 codes."""
    x = np.asarray(x, dtype=np.float64)
    r = np.abs(e4m3_round(x))
    code = np.zeros(r.shape, dtype=np.int64)
    nz = r > 0
    _, ex = np.frexp(r[nz])
    e = ex - 1                                # exact binary exponent of the rounded value
    sub = e < E4M3_MIN_NORMAL_EXP
    rv = r[nz]
    c = np.where(sub,
                 np.rint(rv * 2.0 ** 9).astype(np.int64),                       # m * 2^-9
                 ((e + 7) << 3) | np.rint((np.ldexp(rv, -e) - 1.0) * 8).astype(np.int64))
    code[nz] = c
    sign = np.signbit(x).astype(np.int64)
    return ((sign << 7) | code).astype(np.uint8)


# ---------------------------------------------------------------------------------------
# E8M0
# ---------------------------------------------------------------------------------------

E8M0_BIAS = 127


def e8m0_decode(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    out = np.ldexp(1.0, c - E8M0_BIAS)
    return np.where(c == 0xFF, np.nan, out)


# ---------------------------------------------------------------------------------------
# IEEE half precision (the FP16 tile path; fp16 outputs) and bfloat16 (bf16 outputs)
# ---------------------------------------------------------------------------------------

def fp16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to IEEE binary16 (round-to-nearest-even), returned as float64.

    numpy's float64 -> float16 cast rounds once, to nearest even.
    """
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bfloat16 (8-bit significand, float32's exponent range) once,
    to nearest with ties to even, returned as float64. An attention output requested in bf16
    is the float64 result rounded this way (a single rounding: no float32 step in between).

    Each finite value is split as m 2^e with m in [0.5, 1); m 2^8 is then an exact float64 and
    np.rint rounds it to the nearest integer, ties to even. Below bfloat16's smallest normal
    (2^-126) the step is the subnormal quantum 2^-133; beyond the largest finite value
    (2^128 (1 - 2^-8)) the result is infinite, as IEEE rounding to nearest gives.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    step_exp = np.maximum(e - 8, -133)                       # exponent of one unit in the last place
    out = np.rint(np.ldexp(x, -step_exp)) * np.ldexp(1.0, step_exp)
    big = np.abs(out) >= 2.0 ** 128
    out = np.where(big, np.copysign(np.inf, x), out)
    return np.where(np.isfinite(x), out, x)
