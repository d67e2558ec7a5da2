"""Pins for oracle/formats.py: hand-typed tables, hand-worked roundings, exhaustive
brute-force rounding checks, and torch's own FP8 casts as an independent reference."""
import math

import numpy as np
import pytest
import torch

from oracle import formats as F
from golden_io import pairs


def test_e2m1_table_matches_hand_typed():
    for code, val in pairs("e2m1_codes.txt"):
        c = int(code, 16)
        got = F.E2M1_TABLE[c]
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_e2m1_rounding_hand_worked():
    for x, code in pairs("e2m1_rounding.txt"):
        xv = np.float32(float(x))
        assert int(F.e2m1_encode(np.array([xv]))[0]) == int(code, 16), x


def _nearest_even_brute(a, grid, codes):
    """argmin |a - g| over a magnitude grid; exact ties go to the even code."""
    d = np.abs(grid - a)
    best = d.min()
    cands = [c for c, dd in zip(codes, d) if dd == best]
    if len(cands) > 1:
        cands = [c for c in cands if c % 2 == 0]
    return cands[0]


def test_e2m1_encode_brute_force_sweep():
    mags = F.E2M1_MAGNITUDES
    xs = set()
    for g in mags:
        for dx in (0.0, 1e-3, -1e-3, 0.1, -0.1):
            xs.add(g + dx)
    for i in range(len(mags) - 1):
        mid = 0.5 * (mags[i] + mags[i + 1])
        xs.update({mid, float(np.nextafter(np.float32(mid), np.float32(0))),
                   float(np.nextafter(np.float32(mid), np.float32(10)))})
    xs.update(np.linspace(0, 8, 4001).tolist())
    xs = np.array(sorted(x for x in xs if x >= 0), dtype=np.float32)
    got = F.e2m1_encode(xs)
    for x, c in zip(xs, got):
        want = _nearest_even_brute(min(float(x), 6.0), mags, list(range(8)))
        assert int(c) == want, float(x)
        assert int(F.e2m1_encode(np.array([-x]))[0]) == want | 8


def test_e4m3_table_matches_hand_typed_and_torch():
    for code, val in pairs("e4m3_codes.txt"):
        c = int(code, 16)
        got = F.E4M3_TABLE[c]
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    same = (ref == F.E4M3_TABLE) | (np.isnan(ref) & np.isnan(F.E4M3_TABLE))
    assert same.all()


def test_e8m0_decode_matches_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    got = F.e8m0_decode(np.arange(256))
    same = (ref == got) | (np.isnan(ref) & np.isnan(got))
    assert same.all()
    assert got[127] == 1.0 and got[0] == 2.0 ** -127 and got[254] == 2.0 ** 127


def test_e4m3_rounding_hand_worked():
    for x, code in pairs("e4m3_rounding.txt"):
        assert int(F.e4m3_encode(np.array([np.float32(float(x))]))[0]) == int(code, 16), x


def test_e4m3_round_trip_every_code():
    finite = [c for c in range(256) if not math.isnan(F.E4M3_TABLE[c])]
    vals = F.E4M3_TABLE[finite]
    assert (F.e4m3_encode(vals) == np.array(finite, dtype=np.uint8)).all()


def test_e4m3_midpoints_and_neighbours_brute_force():
    """Every midpoint of neighbouring positive values, and +-1 fp32 ulp around it, against an
    argmin over all 127 non-negative finite codes (ties to the even code)."""
    pos = sorted({float(F.E4M3_TABLE[c]) for c in range(0x7F)})
    grid = np.array(pos)
    codes = [int(F.e4m3_encode(np.array([g]))[0]) for g in pos]
    xs = []
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32(0.5 * (a + b))
        xs += [m, np.nextafter(m, np.float32(0)), np.nextafter(m, np.float32(1e9))]
    xs += [np.float32(448.0), np.float32(463.99), np.float32(464.0), np.float32(500.0)]
    xs = np.array(xs, dtype=np.float32)
    got = F.e4m3_encode(xs)
    for x, c in zip(xs, got):
        want = _nearest_even_brute(min(float(x), 448.0), grid, codes)
        assert int(c) == want, float(x)


def test_e4m3_encode_matches_torch_cast_in_range():
    """torch's float32 -> float8_e4m3fn cast rounds to nearest even; agree for |x| <= 448."""
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-3, 0.05, 1.0, 30.0, 150.0)])
    x = x[x.abs() <= 448]
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode(x.numpy())
    assert (ref == got).all()


def test_fp16_round_is_ieee_half():
    x = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 65504.0, 1e-8, 0.1])
    ref = torch.tensor(x, dtype=torch.float64).to(torch.float16).double().numpy()
    assert (F.fp16_round(x) == ref).all()
    assert F.fp16_round(np.array([1.0 + 2.0 ** -11]))[0] == 1.0          # tie to even


def test_bf16_round_matches_torch_cast_of_float32_values():
    """Values exactly representable in float32 (so torch's float32 -> bfloat16 cast, which
    rounds to nearest even, rounds them once too): the two agree everywhere, subnormals
    included."""
    g = torch.Generator().manual_seed(1)
    x = torch.cat([torch.randn(200000, generator=g) * s for s in (1e-40, 1e-30, 1e-3, 1.0, 3e4, 1e30)])
    ref = x.to(torch.bfloat16).double().numpy()
    assert (F.bf16_round(x.double().numpy()) == ref).all()


def test_bf16_round_hand_worked():
    """Ties to even on both sides, a value just above a tie, and one rounding from float64:
    1 + 2^-8 + 2^-40 rounds up to 1 + 2^-7, while a float32 step first would land on the tie
    1 + 2^-8 and then round down to 1."""
    cases = [(1.0 + 2.0 ** -8, 1.0), (1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -6),
             (-(1.0 + 2.0 ** -8), -1.0), (1.0 + 2.0 ** -8 + 2.0 ** -40, 1.0 + 2.0 ** -7),
             (0.0, 0.0), (2.0 ** -133 * 0.75, 2.0 ** -133), (2.0 ** -133 * 0.5, 0.0),
             (3.0 * 2.0 ** 126 + 2.0 ** 118, 3.0 * 2.0 ** 126)]
    for x, want in cases:
        assert F.bf16_round(np.array([x]))[0] == want, x
    assert np.float32(1.0 + 2.0 ** -8 + 2.0 ** -40) == np.float32(1.0 + 2.0 ** -8)


def test_bf16_round_is_nearest_brute_force():
    """Against the two bracketing bfloat16 values, enumerated from the float32 bit patterns
    around each input: the result is the nearer one, the even one on a tie."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal(3000) * np.exp2(rng.integers(-20, 20, 3000))
    got = F.bf16_round(x)
    for xi, gi in zip(x, got):
        b = int(np.array(abs(xi), dtype=np.float32).view(np.uint32)) & ~0xFFFF
        lo = float(np.array(b, dtype=np.uint32).view(np.float32))
        hi = float(np.array(b + 0x10000, dtype=np.uint32).view(np.float32))
        assert lo <= abs(xi) <= hi
        dl, dh = abs(xi) - lo, hi - abs(xi)
        want = lo if (dl < dh or (dl == dh and (b >> 16) % 2 == 0)) else hi
        assert gi == np.copysign(want, xi), xi
