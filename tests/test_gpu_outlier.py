"""GPU parity of outlier-aware key quantization against the oracle: the smoothing + Hadamard
rotation bit-exact, the scale-searched NVFP4 bit-exact, and attention through the transformed
path matching the oracle and closer to exact attention than the plain path on keys with
outlier channels."""
import math

import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, workloads
from oracle import attention as OA
from oracle import outlier as OO
from oracle import quant as OQ
from helpers import assert_attention_close, f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _lam(q, k):
    """A smoothing vector from the channel ranges (what a calibration run would fix)."""
    qa = q.float().abs().reshape(-1, 128).amax(0)
    ka = k.float().abs().reshape(-1, 128).amax(0)
    return torch.sqrt(ka / qa).float()


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("role", ["q", "k"])
@pytest.mark.parametrize("smooth", [False, True])
def test_smooth_rotate_bit_exact(dtype, role, smooth):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(777, 128, generator=g) * torch.exp(torch.randn(777, 1, generator=g))).to(dtype)
    lam = torch.exp2(torch.rand(128, generator=g) * 4 - 2) if smooth else None
    got = api.qk_smooth_rotate(x.to(DEV), role, None if lam is None else lam.to(DEV))
    want = OO.smooth_rotate(f32(x), None if lam is None else lam.numpy(), role,
                            "bf16" if dtype == torch.bfloat16 else "fp16")
    assert np.array_equal(f32(got), want)


@pytest.mark.parametrize("name", ["prefill_h16_n4096"])
def test_scale_search_bit_exact(name):
    w = workloads.make_prefill(name)
    for x in (w.k, w.q):
        got = api.quantize_nvfp4(x.to(DEV), scale_search=True)
        c, s, t = OO.nvfp4_quantize_searched(f32(x))
        assert np.float32(got.tensor_scale.item()) == t
        gs, gc = got.scales.cpu().numpy(), got.codes.cpu().numpy()
        assert np.array_equal(gs, s), f"scales differ at {np.argwhere(gs != s)[:5]}"
        assert np.array_equal(gc, c), f"codes differ at {np.argwhere(gc != c)[:5]}"


def test_outlier_aware_attention_parity_and_quality():
    """Keys with the workloads' outlier channels: attention on smoothed + rotated Q and K (K with
    the scale search) matches the oracle on those inputs, and is closer to exact attention than
    the plain path."""
    w = workloads.make_prefill("prefill_h16_n4096")
    q, k, v = (t[:, :2, :1024].contiguous() for t in (w.q, w.k, w.v))
    scale = 1 / math.sqrt(128)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    lam = _lam(q, k).to(DEV)
    qr, kr = api.qk_smooth_rotate(qd, "q", lam), api.qk_smooth_rotate(kd, "k", lam)
    q4, k4 = api.quantize_nvfp4(qr), api.quantize_nvfp4(kr, scale_search=True)
    v8 = api.quantize_mxfp8_v(vd)
    out_t = f32(api.attn_qk4v8_fwd(q4, k4, v8, True, scale, torch.float32))
    out_p = f32(api.qk4v8_attention(qd, kd, vd, True, scale, out_dtype=torch.float32))
    assert api.check_status() == 0
    ref = np.zeros_like(out_t)
    exact = np.zeros_like(out_t)
    # the oracle's own transform of the CPU inputs (bit-exact with the kernel's, tested above)
    lam_np = lam.cpu().numpy()
    qr_o = OO.smooth_rotate(f32(q), lam_np, "q", "bf16")
    kr_o = OO.smooth_rotate(f32(k), lam_np, "k", "bf16")
    sq, sk = OQ.nvfp4_tensor_scale(qr_o), OQ.nvfp4_tensor_scale(kr_o)
    for h in range(2):
        qh = OQ.nvfp4_dequantize(*OQ.nvfp4_quantize(qr_o[0, h], tensor_scale=sq))
        kh = OQ.nvfp4_dequantize(*OO.nvfp4_quantize_searched(kr_o[0, h], tensor_scale=sk))
        vc, vs = OQ.mxfp8_quantize_v(f32(v[0, h]))
        vh = OQ.mxfp8_dequantize_v(vc, vs, 1024)
        ref[0, h] = OA.attention_head(qh, kh, vh, True, scale)[0]
        exact[0, h] = OA.exact_attention(f32(q[0, h]).astype(np.float64), f32(k[0, h]).astype(np.float64),
                                         f32(v[0, h]).astype(np.float64), True, scale)
    assert_attention_close(out_t, ref, "outlier-aware")
    e_p, e_t = np.abs(out_p - exact).mean(), np.abs(out_t - exact).mean()
    assert e_t < e_p, (e_p, e_t)
