"""GPU parity of the quantize kernels against the oracle: bit-exact codes, scales and tensor
scales on the workloads' Q/K/V, ragged shapes, and exhaustive sweeps of every fp16 input
through the E2M1 element, E4M3 block-scale and E4M3 V-element conversions."""
import numpy as np
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, workloads
from oracle import formats as OF
from oracle import quant as OQ
from helpers import f32

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _nvfp4_equal(x_cpu, tensor_scale=None, want_fp16=False):
    g = api.quantize_nvfp4(x_cpu.to(DEV), tensor_scale=tensor_scale, want_fp16=want_fp16)
    c, s, t = OQ.nvfp4_quantize(f32(x_cpu), tensor_scale=tensor_scale)
    gc, gs = g.codes.cpu().numpy(), g.scales.cpu().numpy()
    assert np.array_equal(gs, s), f"scales differ at {np.argwhere(gs != s)[:5]}"
    assert np.array_equal(gc, c), f"codes differ at {np.argwhere(gc != c)[:5]}"
    assert np.float32(g.tensor_scale.item()) == t
    if want_fp16:
        assert np.array_equal(g.fp16.cpu().numpy(), OF.fp16_round(f32(x_cpu)).astype(np.float16))
    return g


@pytest.mark.parametrize("name", ["tiny_prefill", "prefill_h16_n4096"])
def test_nvfp4_workload_q_k_bit_exact(name):
    w = workloads.make_prefill(name)
    _nvfp4_equal(w.q)
    _nvfp4_equal(w.k, want_fp16=True)


@pytest.mark.parametrize("shape,dtype", [((1000, 64), torch.bfloat16), ((3, 37, 128), torch.float16),
                                         ((1, 16), torch.bfloat16)])
def test_nvfp4_ragged_shapes(shape, dtype):
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(shape, generator=g) * torch.rand(shape[:-1] + (1,), generator=g) * 7).to(dtype)
    _nvfp4_equal(x)
    _nvfp4_equal(x, tensor_scale=0.0625)


@pytest.mark.parametrize("ts", [None, 2.0 ** -120, 2.0 ** -95, 0.3, 1.7e5, 2.0 ** 85, 2.0 ** 100])
def test_nvfp4_division_across_scale_ranges(ts):
    """Element quotients x / (s_b s_t) with the divisor on both sides of the bounds of the
    kernel's fast division (2^-90, 2^90) and far inside them, non-power-of-two scales, block
    magnitudes spread over 24 octaves around the scale: codes bit-exact against the oracle."""
    g = torch.Generator().manual_seed(17)
    base = 1.0 if ts is None else ts
    x = torch.randn(8192, 64, generator=g, dtype=torch.float64)
    octave = torch.randint(-12, 13, (8192, 1), generator=g).double()
    x = (x * base * 1.37 * torch.pow(2.0, octave)).to(torch.bfloat16)
    _nvfp4_equal(x, tensor_scale=ts)


def test_nvfp4_zero_tensor():
    g = api.quantize_nvfp4(torch.zeros(4, 64, dtype=torch.bfloat16, device=DEV))
    assert g.tensor_scale.item() == 1.0 and not g.codes.any() and not g.scales.any()


def _all_fp16_values(lo_bits, hi_bits):
    return torch.arange(lo_bits, hi_bits, dtype=torch.int32).to(torch.int16).view(torch.float16)


def test_e2m1_conversion_exhaustive_fp16():
    """Tensor scale 2^-8 and a leading 6 in every block give s_b = 256, den = 1: each code is
    E2M1 of the raw fp16 value. Every fp16 value in [-8, 8] (both signs, zeros) is swept."""
    pos = _all_fp16_values(0x0000, 0x4801)                  # 0 .. 8
    vals = torch.cat([pos, -pos])
    n = vals.numel()
    nb = (n + 14) // 15
    x = torch.zeros(nb, 16, dtype=torch.float16)
    x[:, 0] = 6.0
    flat = torch.zeros(nb * 15, dtype=torch.float16)
    flat[:n] = vals
    x[:, 1:] = flat.view(nb, 15)
    _nvfp4_equal(x, tensor_scale=2.0 ** -8)


def test_e4m3_block_scale_exhaustive_fp16():
    """Every positive finite fp16 value as a block amax, with tensor scale 2^-4: the block
    scale is E4M3(amax / 6 / 2^-4) across the whole E4M3 range, subnormals and saturation."""
    amax = _all_fp16_values(0x0001, 0x7C00)
    x = torch.zeros(amax.numel(), 16, dtype=torch.float16)
    x[:, 3] = amax
    x[:, 7] = -amax / 3
    _nvfp4_equal(x, tensor_scale=2.0 ** -4)


def _all_bf16_values(lo_bits, hi_bits):
    return torch.arange(lo_bits, hi_bits, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)


@pytest.mark.parametrize("ts", [None, 0.37, 2.0 ** -70, 3.1e17])
def test_block_scale_and_codes_exhaustive_bf16(ts):
    """Every positive finite bf16 value (subnormals included) as a block's largest magnitude,
    with the other elements of the block at -1/3, 5/7 and 1/11 of it: the block scale
    E4M3(amax_b / 6 / s_t) and every element code, bit-exact against the oracle, for the
    computed tensor scale and fixed scales with ordinary, tiny and huge values (both sides of
    the exponent bounds of the kernels' fast division). Checked through the per-tensor kernel
    and the fused Q/K/V kernel."""
    amax = _all_bf16_values(0x0001, 0x7F80)
    x = torch.zeros(amax.numel(), 16, dtype=torch.bfloat16)
    x[:, 3] = amax
    x[:, 7] = (-amax.double() / 3).to(torch.bfloat16)
    x[:, 9] = (amax.double() * 5 / 7).to(torch.bfloat16)
    x[:, 14] = (amax.double() / 11).to(torch.bfloat16)
    assert torch.isfinite(x.float()).all()
    _nvfp4_equal(x, tensor_scale=ts)
    if ts is None:
        # the same 16-element blocks, 128 to a row (the fused call's head dimension)
        xq = torch.cat([x, torch.zeros(1, 16, dtype=torch.bfloat16)]).reshape(-1, 128)
        xk = x[:4096].reshape(-1, 128)
        v = torch.zeros(1, 128, 128, dtype=torch.bfloat16)
        q4, k4, _ = api.quantize_qkv(xq.to(DEV), xk.to(DEV), v.to(DEV))
        for g, xx in ((q4, xq), (k4, xk)):
            c, sc, t = OQ.nvfp4_quantize(f32(xx))
            assert np.array_equal(g.scales.cpu().numpy(), sc) and np.array_equal(g.codes.cpu().numpy(), c)
            assert np.float32(g.tensor_scale.item()) == t


def _mxfp8_equal(v_cpu, want_fp16=False):
    g = api.quantize_mxfp8_v(v_cpu.to(DEV), want_fp16=want_fp16)
    c, s = OQ.mxfp8_quantize_v(f32(v_cpu))
    gc, gs = g.codes.cpu().numpy(), g.scales.cpu().numpy()
    assert np.array_equal(gs, s), f"scales differ at {np.argwhere(gs != s)[:5]}"
    assert np.array_equal(gc, c), f"codes differ at {np.argwhere(gc != c)[:5]}"
    if want_fp16:
        n = v_cpu.shape[-2]
        ref = np.zeros(gc.shape, dtype=np.float16)
        ref[..., :n] = np.swapaxes(OF.fp16_round(f32(v_cpu)), -1, -2)
        assert np.array_equal(g.fp16.cpu().numpy(), ref)


@pytest.mark.parametrize("name", ["tiny_prefill", "prefill_h16_n4096"])
def test_mxfp8_workload_v_bit_exact(name):
    w = workloads.make_prefill(name)
    _mxfp8_equal(w.v, want_fp16=True)


@pytest.mark.parametrize("n,d", [(1, 128), (300, 64), (129, 128)])
def test_mxfp8_ragged(n, d):
    g = torch.Generator().manual_seed(n)
    v = (torch.randn(3, n, d, generator=g) * torch.rand(3, 1, d, generator=g) * 50).to(torch.bfloat16)
    _mxfp8_equal(v, want_fp16=True)


def test_e4m3_element_conversion_exhaustive_fp16():
    """Groups whose first token is 480 have e = 0 (480 saturates to 448); the other 31 tokens
    sweep every fp16 value in [-480, 480], so each code is E4M3 of the raw value."""
    pos = _all_fp16_values(0x0000, 0x5F81)                  # 0 .. 480
    vals = torch.cat([pos, -pos])
    n = vals.numel()
    ng = (n + 30) // 31
    ng = (ng + 3) // 4 * 4
    d = 64
    col = torch.zeros(ng, 32, dtype=torch.float16)
    col[:, 0] = 480.0
    flat = torch.zeros(ng * 31, dtype=torch.float16)
    flat[:n] = vals
    col[:, 1:] = flat.view(ng, 31)
    tokens = col.reshape(-1)                                # ng*32 tokens, one channel
    v = torch.zeros(1, tokens.numel(), d, dtype=torch.float16)
    v[0, :, 5] = tokens
    v[0, :, 60] = -tokens
    _mxfp8_equal(v)


@pytest.mark.parametrize("shape,dtype", [((16, 4096, 128), torch.bfloat16), ((3, 37, 64), torch.float16),
                                         ((1, 16), torch.bfloat16)])
def test_nvfp4_residual_bit_exact(shape, dtype):
    """The second tensor of dual-residual quantization: codes and scales bit-exact."""
    g = torch.Generator().manual_seed(sum(shape))
    x = (torch.randn(shape, generator=g) * torch.rand(shape[:-1] + (1,), generator=g) * 7).to(dtype)
    q1, q2 = api.quantize_nvfp4_dual(x.to(DEV))
    c1, s1, c2, s2, t = OQ.nvfp4_dual_quantize(f32(x))
    assert np.array_equal(q1.codes.cpu().numpy(), c1) and np.array_equal(q1.scales.cpu().numpy(), s1)
    gs, gc = q2.scales.cpu().numpy(), q2.codes.cpu().numpy()
    assert np.array_equal(gs, s2), f"scales differ at {np.argwhere(gs != s2)[:5]}"
    assert np.array_equal(gc, c2), f"codes differ at {np.argwhere(gc != c2)[:5]}"
    assert q2.tensor_scale is q1.tensor_scale and np.float32(q1.tensor_scale.item()) == t


def _check_qkv(q, k, v, want_fp16=False):
    """quantize_qkv (two launches) against the oracle, bit for bit, and against the per-tensor
    calls (identical outputs); with ``want_fp16`` also V's fp16 copy (Q and K get none)."""
    q4, k4, v8 = api.quantize_qkv(q.to(DEV), k.to(DEV), v.to(DEV), want_fp16_v=want_fp16)
    for g, x in ((q4, q), (k4, k)):
        c, s, t = OQ.nvfp4_quantize(f32(x))
        gc, gs = g.codes.cpu().numpy(), g.scales.cpu().numpy()
        assert np.array_equal(gs, s), f"scales differ at {np.argwhere(gs != s)[:5]}"
        assert np.array_equal(gc, c), f"codes differ at {np.argwhere(gc != c)[:5]}"
        assert np.float32(g.tensor_scale.item()) == t
        assert g.fp16 is None
    n = v.shape[-2]
    vc, vs = OQ.mxfp8_quantize_v(f32(v))
    npad = v8.codes.shape[-1]
    assert np.array_equal(v8.codes.cpu().numpy(), vc)
    assert np.array_equal(v8.scales.cpu().numpy(), vs)
    if want_fp16:
        r16 = np.zeros(v8.fp16.shape, dtype=np.float16)
        r16[..., :n] = np.swapaxes(OF.fp16_round(f32(v)), -1, -2)
        assert np.array_equal(v8.fp16.cpu().numpy(), r16)
    # the per-tensor entry points give the same bytes
    sq, sk, sv = api.quantize_nvfp4(q.to(DEV)), api.quantize_nvfp4(k.to(DEV)), api.quantize_mxfp8_v(v.to(DEV))
    assert torch.equal(sq.codes, q4.codes) and torch.equal(sq.scales, q4.scales)
    assert torch.equal(sk.codes, k4.codes) and torch.equal(sk.tensor_scale, k4.tensor_scale)
    assert torch.equal(sv.codes, v8.codes) and torch.equal(sv.scales, v8.scales)
    assert npad == (n + 127) // 128 * 128


@pytest.mark.parametrize("name", ["tiny_prefill", "prefill_h16_n4096"])
def test_qkv_workload_bit_exact(name):
    w = workloads.make_prefill(name)
    _check_qkv(w.q, w.k, w.v)


@pytest.mark.parametrize("hq,hkv,n,d,dtype,fp16", [(4, 1, 1000, 128, torch.bfloat16, False),
                                                  (3, 3, 77, 64, torch.float16, True),
                                                  (8, 2, 300, 128, torch.bfloat16, True)])
def test_qkv_ragged_shapes(hq, hkv, n, d, dtype, fp16):
    """Chunk tails (blocks not a multiple of the 1024-block chunk), V tails (tokens not a
    multiple of 128), head_dim 64, fp16 inputs, the optional fp16 copies, and Q/K size ratios of
    1, 3 and 4."""
    g = torch.Generator().manual_seed(n + d)
    q = (torch.randn(1, hq, n, d, generator=g) * 3).to(dtype)
    k = (torch.randn(1, hkv, n, d, generator=g) * torch.rand(1, hkv, n, 1, generator=g) * 9).to(dtype)
    v = torch.randn(1, hkv, n, d, generator=g).to(dtype)
    _check_qkv(q, k, v, want_fp16=fp16)
