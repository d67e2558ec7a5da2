"""Pins for oracle/paged.py: pages placed at shuffled physical ids read back bit-identical,
and decode through the gathered pages equals decode on the dense quantized sequence."""
import numpy as np

from oracle import attention as A
from oracle import paged as P
from oracle import quant as Q


def test_pages_round_trip_through_shuffled_table():
    rng = np.random.default_rng(0)
    lens = [1, 64, 65, 300]
    hkv, d = 2, 64
    seqs = [(rng.standard_normal((n, hkv, d)).astype(np.float32),
             rng.standard_normal((n, hkv, d)).astype(np.float32)) for n in lens]
    n_pages = [(n + 63) // 64 for n in lens]
    total = sum(n_pages)
    perm = rng.permutation(total)
    kp = np.zeros((total, hkv, 64, d // 2), np.uint8); ksp = np.zeros((total, hkv, 64, d // 16), np.uint8)
    vp = np.zeros((total, hkv, d, 64), np.uint8); vsp = np.zeros((total, hkv, d, 2), np.uint8)
    table = np.full((len(lens), max(n_pages)), -1)
    off = 0
    dense = []
    for s, (k, v) in enumerate(seqs):
        kc, ks, vc, vs = P.quantize_sequence(k, v, 0.0625)
        dense.append((kc, ks, vc, vs))
        pages = P.sequence_pages(kc, ks, vc, vs, lens[s])
        ids = perm[off:off + n_pages[s]]
        table[s, :n_pages[s]] = ids
        for j, i in enumerate(ids):
            kp[i], ksp[i], vp[i], vsp[i] = pages[0][j], pages[1][j], pages[2][j], pages[3][j]
        off += n_pages[s]
    for s, n in enumerate(lens):
        kc, ks, vc, vs = P.gather_sequence(kp, ksp, vp, vsp, table[s], n)
        dk, dks, dvc, dvs = dense[s]
        assert np.array_equal(kc, dk) and np.array_equal(ks, dks)
        npad = (n + 63) // 64 * 64
        assert np.array_equal(vc, dvc[:, :, :npad]) and np.array_equal(vs, dvs[:, :, :npad // 32])
        vh = Q.mxfp8_dequantize_v(vc, vs, n)
        kh = Q.nvfp4_dequantize(kc, ks, 0.0625)
        q = rng.standard_normal((2, d))
        o, _ = A.decode_rows(q, kh[0], vh[0], n, 0.125, 128)
        assert np.all(np.isfinite(o))
