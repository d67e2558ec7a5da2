"""Pins for oracle/quant.py: hand-worked blocks, brute force over the code space, exact
power-of-two invariances, and closed-form facts of the two-level NVFP4 scaling."""
import numpy as np
import pytest
import torch

from oracle import formats as F
from oracle import quant as Q
from golden_io import keyed

F32 = np.float32


def test_nvfp4_hand_worked_blocks():
    g = keyed("nvfp4_blocks.txt")
    x = np.array([float(t) for t in g["x"]], dtype=F32)[None, :]
    codes, scales, s_t = Q.nvfp4_quantize(x)
    assert s_t == F32(float(g["tensor_scale"][0]))
    assert codes[0].tolist() == [int(t, 16) for t in g["codes"]]
    assert scales[0].tolist() == [int(t, 16) for t in g["scales"]]


def _brute_nvfp4_block(xb, s_t):
    """Independent per-block reference: choose the E4M3 scale code whose value is nearest to
    fl32(fl32(amax/6)/s_t) by scanning all 127 non-negative finite codes, then each element
    code by scanning all 16 E2M1 codes for the nearest multiple of den (ties: even code)."""
    amax = F32(np.max(np.abs(xb)))
    target = float(F32(F32(amax / F32(6)) / s_t))
    best, best_c = None, None
    for c in range(0x7F):
        val = F.E4M3_TABLE[c]
        dist = abs(min(target, 448.0) - val)
        if best is None or dist < best or (dist == best and c % 2 == 0):
            best, best_c = dist, c
    sb = F32(F.E4M3_TABLE[best_c])
    if sb == 0:
        return [0] * len(xb), best_c
    den = F32(sb * s_t)
    out = []
    for x in xb:
        r = float(F32(F32(x) / den))
        rr = min(abs(r), 6.0)
        bd, bc = None, None
        for c in range(8):
            dist = abs(rr - F.E2M1_MAGNITUDES[c])
            if bd is None or dist < bd or (dist == bd and c % 2 == 0):
                bd, bc = dist, c
        out.append(bc | (8 if np.signbit(r) else 0))
    return out, best_c


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_nvfp4_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((6, 64)) * rng.choice([1e-3, 1.0, 50.0], size=(6, 1))).astype(F32)
    x[2, 16:32] = 0.0
    x[3, 0] = 300.0
    codes, scales, s_t = Q.nvfp4_quantize(x)
    un = Q.nvfp4_unpack(codes)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            want, want_sc = _brute_nvfp4_block(x[r, 16 * b:16 * b + 16], s_t)
            assert un[r, 16 * b:16 * b + 16].tolist() == want
            assert scales[r, b] == want_sc


def test_nvfp4_tensor_max_block_has_scale_448_and_code_6():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((8, 128)).astype(F32)
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    codes, scales, s_t = Q.nvfp4_quantize(x)
    assert F.E4M3_TABLE[scales[i[0], i[1] // 16]] == 448.0
    assert Q.nvfp4_unpack(codes)[i] & 7 == 7
    assert np.all(F.E4M3_TABLE[scales] <= 448.0)


@pytest.mark.parametrize("k", [-20, -3, 1, 7])
def test_nvfp4_power_of_two_invariance(k):
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((4, 96)) * 3).astype(F32)
    c0, s0, t0 = Q.nvfp4_quantize(x)
    c1, s1, t1 = Q.nvfp4_quantize((x * F32(2.0 ** k)).astype(F32))
    assert (c0 == c1).all() and (s0 == s1).all()
    assert t1 == F32(t0 * F32(2.0 ** k))


def test_nvfp4_error_within_half_step_of_block_grid():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal((16, 128)) * 2).astype(F32)
    codes, scales, s_t = Q.nvfp4_quantize(x)
    xh = Q.nvfp4_dequantize(codes, scales, s_t)
    den = F.e4m3_decode(scales).repeat(16, axis=1) * np.float64(s_t)
    # grid spacing around |x|/den: 0.5 below 2, 1 in [2,4), 2 in [4,6]
    r = np.abs(x / den)
    step = np.where(r < 2, 0.5, np.where(r < 4, 1.0, 2.0))
    assert np.all(np.abs(xh - x) <= 0.5 * step * den * (1 + 1e-6) + 1e-30)


def test_nvfp4_zero_tensor_and_given_scale():
    codes, scales, s_t = Q.nvfp4_quantize(np.zeros((2, 32), F32))
    assert s_t == 1.0 and not codes.any() and not scales.any()
    x = np.full((1, 16), 3.0, F32)
    codes, scales, s_t = Q.nvfp4_quantize(x, tensor_scale=0.0625)
    # 3/6/0.0625 = 8 -> scale 8.0 (0x50); den = 0.5; 3/0.5 = 6 -> code 7
    assert s_t == F32(0.0625) and scales[0, 0] == 0x50 and (Q.nvfp4_unpack(codes) == 7).all()


def test_mxfp8_hand_worked_group():
    g = keyed("mxfp8_group.txt")
    v = np.zeros((64, 1), F32)
    vals = [float(t) for t in g["v"]]
    v[:len(vals), 0] = vals
    codes, scales = Q.mxfp8_quantize_v(v)
    assert codes.shape == (1, 128) and scales.shape == (1, 4)
    assert scales[0].tolist() == [int(t, 16) for t in g["scales"]]
    assert codes[0, :len(vals)].tolist() == [int(t, 16) for t in g["codes"]]
    assert not codes[0, len(vals):].any()


def test_mxfp8_brute_force_and_exponent_rule():
    rng = np.random.default_rng(7)
    v = (rng.standard_normal((3, 100, 8)) * rng.choice([1e-4, 1.0, 40.0], size=(3, 1, 1))).astype(F32)
    codes, scales = Q.mxfp8_quantize_v(v)
    assert codes.shape == (3, 8, 128) and scales.shape == (3, 8, 4)
    pos = sorted({float(F.E4M3_TABLE[c]) for c in range(0x7F)})
    grid = np.array(pos)
    for b in range(3):
        for c in range(8):
            for gi in range(4):
                grp = v[b, 32 * gi:min(32 * gi + 32, 100), c].astype(np.float64)
                if grp.size == 0 or not np.any(grp):
                    assert scales[b, c, gi] == 127
                    continue
                e = int(scales[b, c, gi]) - 127
                amax = np.abs(grp).max()
                assert 256.0 <= amax / 2.0 ** e < 512.0        # floor(log2 amax) - e == 8
                for j, x in enumerate(grp):
                    r = min(abs(x) / 2.0 ** e, 448.0)
                    best = np.abs(grid - r).min()
                    cand = [i for i, g_ in enumerate(grid) if abs(g_ - r) == best]
                    want_val = grid[cand[0]] if len(cand) == 1 else \
                        [grid[i] for i in cand if int(F.e4m3_encode(np.array([grid[i]]))[0]) % 2 == 0][0]
                    got = F.E4M3_TABLE[codes[b, c, 32 * gi + j]]
                    assert abs(got) == want_val and (got == 0 or np.sign(got) == np.sign(x))
    assert not codes[..., 100:].any()


@pytest.mark.parametrize("k", [-9, 2, 30])
def test_mxfp8_power_of_two_invariance(k):
    rng = np.random.default_rng(1)
    v = rng.standard_normal((2, 64, 16)).astype(F32)
    c0, s0 = Q.mxfp8_quantize_v(v)
    c1, s1 = Q.mxfp8_quantize_v((v * F32(2.0 ** k)).astype(F32))
    assert (c0 == c1).all()
    live = slice(0, 2)                      # groups 2, 3 are padding (scale code 127 always)
    assert (s1[..., live].astype(int) == s0[..., live].astype(int) + k).all()
    assert (s1[..., 2:] == 127).all()


def test_mxfp8_dequant_layout_round_trip():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((2, 70, 16)).astype(F32)
    codes, scales = Q.mxfp8_quantize_v(v)
    vh = Q.mxfp8_dequantize_v(codes, scales, 70)
    assert vh.shape == v.shape
    # half an E4M3 ulp: relative 2^-4 for normals, absolute 2^(e-10) in the subnormal range;
    # values above 448 * 2^e saturate to 448 * 2^e
    e = scales.astype(np.int64) - 127                          # [2, 16, 4]
    step = np.ldexp(1.0, np.repeat(e, 32, axis=-1)[..., :70])  # 2^e per element, [2, 16, 70]
    step = np.swapaxes(step, -1, -2)
    vv = v.astype(np.float64)
    sat = np.abs(vv) > 448.0 * step
    bound = np.maximum(np.abs(vv) * 2.0 ** -4, step * 2.0 ** -10)
    err = np.abs(vh - vv)
    assert np.all(err[~sat] <= bound[~sat])
    assert np.all(np.abs(vh[sat]) == 448.0 * step[sat])


# ---- dual-residual NVFP4 (Q = Q1 + Q2) ----

def test_dual_residual_hand_worked_block():
    """Fixed s_t = 1, block [6, 1.3, 0, ...]: Q1 keeps 6 and rounds 1.3 to 1.5 (s_b = 1).
    The residual fl32(1.3 - 1.5) = -0.2 has amax/6 = 0.0333, which E4M3 rounds to
    1.125 * 2^-5 = 0.03515625 (its neighbours 0.03125 and 0.03515625); -0.2 / 0.03515625 =
    -5.69 rounds to E2M1 -6, so Q2 holds -0.2109375 and Q1 + Q2 = 1.2890625."""
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0], x[0, 1] = 6.0, 1.3
    c1, s1, c2, s2, s_t = Q.nvfp4_dual_quantize(x, tensor_scale=1.0)
    x1 = Q.nvfp4_dequantize(c1, s1, s_t)
    x2 = Q.nvfp4_dequantize(c2, s2, s_t)
    assert x1[0, 0] == 6.0 and x1[0, 1] == 1.5
    assert F.e4m3_decode(s2)[0, 0] == 0.03515625
    assert x2[0, 1] == -0.2109375 and x2[0, 0] == 0.0
    assert x1[0, 1] + x2[0, 1] == 1.2890625


def test_dual_residual_is_zero_on_the_grid():
    """Values exactly on the NVFP4 grid leave no residual: every Q2 code and scale is 0."""
    rng = np.random.default_rng(1)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], dtype=np.float32)
    x = rng.choice(grid, (64, 32)) * rng.choice([-1, 1], (64, 32)).astype(np.float32)
    x[:, 0] = 6.0                                       # every block's scale is exactly 1
    x[:, 16] = 6.0
    c1, s1, c2, s2, _ = Q.nvfp4_dual_quantize(x, tensor_scale=1.0 / 448)
    assert not (Q.nvfp4_unpack(c2) & 7).any() and not s2.any()


def test_residual_brute_force_fp32_steps():
    """The residual, element by element with numpy float32 scalars."""
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((3, 32)) * 5).astype(np.float32)
    c1, s1, s_t = Q.nvfp4_quantize(x)
    r = Q.nvfp4_residual(x, c1, s1, s_t)
    codes = Q.nvfp4_unpack(c1)
    for i in range(3):
        for j in range(32):
            den = np.float32(np.float32(F.e4m3_decode(s1[i, j // 16])) * s_t)
            d = np.float32(np.float32(F.e2m1_decode(codes[i, j])) * den)
            assert r[i, j] == np.float32(x[i, j] - d)


def test_dual_residual_cuts_logit_error():
    """Relative logit error |(q - q_hat) . k| / |q . k| over many query/key pairs: the second
    FP4 tensor cuts it several fold (the page reports 60 % -> 1 % on real queries)."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((256, 128)).astype(np.float32)
    q[:, :4] *= 10.0                                   # outlier channels
    k = rng.standard_normal((256, 128))
    c1, s1, c2, s2, s_t = Q.nvfp4_dual_quantize(q)
    q1 = Q.nvfp4_dequantize(c1, s1, s_t)
    q12 = q1 + Q.nvfp4_dequantize(c2, s2, s_t)
    ref = q.astype(np.float64) @ k.T
    e1 = np.linalg.norm((q1 - q) @ k.T) / np.linalg.norm(ref)
    e2 = np.linalg.norm((q12 - q) @ k.T) / np.linalg.norm(ref)
    assert e2 < e1 / 5, (e1, e2)
