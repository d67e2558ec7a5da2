"""Pins for oracle/outlier.py: the butterfly Hadamard against the Sylvester matrix, exact logit
invariance of smoothing + rotation, the scale search against a brute-force argmin, and the
logit error on keys with outlier channels."""
import numpy as np
import scipy.linalg

from oracle import formats as F
from oracle import outlier as O
from oracle import quant as Q


def test_butterflies_equal_the_sylvester_matrix_and_square_to_128():
    rng = np.random.default_rng(0)
    x = rng.integers(-50, 50, (8, 128)).astype(np.float32)      # exact in float32 throughout
    h = scipy.linalg.hadamard(128)
    assert np.array_equal(O.hadamard_rows(x), (x.astype(np.float64) @ h).astype(np.float32))
    assert np.array_equal(O.hadamard_rows(O.hadamard_rows(x)), 128 * x)


def test_smoothing_and_rotation_keep_every_logit():
    """Before the final 16-bit rounding, (q lam) H 2^-3 . (k / lam) H 2^-4 = q . k up to float32
    rounding of the intermediate steps."""
    rng = np.random.default_rng(1)
    q = rng.standard_normal((16, 128)).astype(np.float32)
    k = rng.standard_normal((64, 128)).astype(np.float32)
    lam = np.exp2(rng.uniform(-2, 2, 128)).astype(np.float32)
    qs = O.hadamard_rows((q * lam).astype(np.float32)) * np.float32(2.0 ** -3)
    ks = O.hadamard_rows((k / lam).astype(np.float32)) * np.float32(2.0 ** -4)
    ref = q.astype(np.float64) @ k.T.astype(np.float64)
    got = qs.astype(np.float64) @ ks.T.astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref))


def test_bf16_round_ties_to_even():
    x = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.0 + 2.0 ** -9, -2.5], dtype=np.float32)
    want = np.array([1.0, 1.0, 1.0 + 4 * 2.0 ** -8, 1.0, -2.5], dtype=np.float32)
    assert np.array_equal(O.bf16_round(x), want)


def _block_error(x, code, s_t):
    den = np.float32(np.float32(F.e4m3_decode(np.array([code], np.uint8))[0]) * s_t)
    e2 = F.e2m1_encode((x / den).astype(np.float32))
    vals = F.e2m1_decode(e2).astype(np.float32)
    err = np.float32(0)
    for i in range(16):
        d = np.float32(x[i] - np.float32(vals[i] * den))
        err = np.float32(err + np.float32(d * d))
    return err


def test_scale_search_is_the_brute_force_argmin():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((40, 16)) * np.exp2(rng.uniform(-3, 3, (40, 1)))).astype(np.float32)
    x[::5, 3] *= 9.0                                   # outliers inside some blocks
    s_t = np.float32(0.01)
    packed, scales, _ = O.nvfp4_quantize_searched(x, tensor_scale=s_t)
    plain_packed, plain_scales, _ = Q.nvfp4_quantize(x, tensor_scale=s_t)
    for b in range(40):
        c0 = int(plain_scales[b, 0])
        cands = [c for c in (c0, c0 - 1, c0 - 2, c0 + 1) if 1 <= c <= 126]
        errs = [_block_error(x[b], c, s_t) for c in cands]
        best = cands[int(np.argmin(errs))]                # first minimum = earlier candidate
        assert scales[b, 0] == best
        assert _block_error(x[b], best, s_t) <= _block_error(x[b], c0, s_t)
        if best == c0:
            assert np.array_equal(packed[b], plain_packed[b])


def test_outlier_keys_lose_less_with_smoothing_rotation_and_search():
    """Keys like the workloads' (per-channel mean, four channels x10): relative logit error of
    NVFP4 Q and K, plain against smoothed + rotated + searched (lam from the channel ranges)."""
    rng = np.random.default_rng(3)
    d = 128
    k = rng.standard_normal((512, d)) + rng.normal(0, 0.5, d)
    k[:, [3, 40, 77, 101]] *= 10.0
    q = rng.standard_normal((64, d))
    ref = q @ k.T

    def logits(qh, kh):
        return np.linalg.norm(qh @ kh.T - ref) / np.linalg.norm(ref)

    deq = lambda t, fn=Q.nvfp4_quantize: Q.nvfp4_dequantize(*fn(t))
    plain = logits(deq(q.astype(np.float32)), deq(k.astype(np.float32)))
    lam = np.sqrt(np.abs(k).max(axis=0) / np.abs(q).max(axis=0)).astype(np.float32)
    qs = O.smooth_rotate(q, lam, "q", "bf16")
    ks = O.smooth_rotate(k, lam, "k", "bf16")
    tr = logits(deq(qs), deq(ks, O.nvfp4_quantize_searched))
    assert tr < plain / 1.5, (plain, tr)
