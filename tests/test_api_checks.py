"""Host-side checks of the torch binding, without a GPU: every buffer is checked against the
sizes the library will be given before any call. Buffers shaped as the binding's own
producers shape them (and as the GPU tests pass them) get past the shape and dtype checks and
stop only at the device check here; a buffer of another shape, dtype or layout is refused."""
import pytest
import torch

from bit_block_scaled_nvfp4_b200 import api, paged

DEVICE_ERR = "contiguous tensors on one CUDA device"


def _prefill(B, Hq, Hkv, Nq, Nk, D, fp16=False):
    q = api._nvfp4_empty((B, Hq, Nq, D), "cpu")
    k = api._nvfp4_empty((B, Hkv, Nk, D), "cpu")
    v = api._mxfp8_empty((B, Hkv, Nk, D), "cpu", fp16)
    return q, k, v


def _inputs16(B, Hq, Hkv, Nq, Nk, D, dtype=torch.bfloat16):
    return torch.empty(B, Hq, Nq, D, dtype=dtype), torch.empty(B, Hkv, Nk, D, dtype=dtype)


def _bitmap(B, Hq, N):
    t = (N + 127) // 128
    return torch.zeros(B * Hq, t, t, dtype=torch.uint8)


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,D", [
    (1, 16, 16, 4096, 4096, 128), (1, 32, 8, 32768, 32768, 128), (2, 4, 2, 700, 700, 128),
    (1, 2, 1, 300, 900, 64), (3, 6, 3, 1, 129, 64), (1, 2, 2, 128, 1, 128)])
def test_fwd_accepts_producer_shapes(B, Hq, Hkv, Nq, Nk, D):
    q, k, v = _prefill(B, Hq, Hkv, Nq, Nk, D)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.attn_qk4v8_fwd(q, k, v, True)
    q2 = api._nvfp4_empty((B, Hq, Nq, D), "cpu")
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.attn_qk4v8_fwd(q, k, v, True, q2=q2, underflow_aware=True)


@pytest.mark.parametrize("N", [128, 700, 16384])
def test_fwd_fp16_tiles_accept_producer_shapes(N):
    q, k, v = _prefill(1, 4, 2, N, N, 128, fp16=True)
    for dt in (torch.bfloat16, torch.float16):
        q16, k16 = _inputs16(1, 4, 2, N, N, 128, dt)
        with pytest.raises(ValueError, match=DEVICE_ERR):
            api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, N), q16=q16, k16=k16)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.tile_score_select(q, k, True, 500)


def test_fwd_refuses_mismatched_buffers():
    q, k, v = _prefill(1, 4, 2, 300, 300, 128)
    short_v = api._mxfp8_empty((1, 2, 200, 128), "cpu")            # V of fewer tokens than K
    with pytest.raises(ValueError, match="v.codes"):
        api.attn_qk4v8_fwd(q, k, short_v, True)
    k_other_d = api._nvfp4_empty((1, 2, 300, 64), "cpu")
    with pytest.raises(ValueError, match="k.codes"):
        api.attn_qk4v8_fwd(q, k_other_d, v, True)
    bad_scales = api.NVFP4Tensor(q.codes, q.scales[..., :4].contiguous(), q.tensor_scale)
    with pytest.raises(ValueError, match="q.scales"):
        api.attn_qk4v8_fwd(bad_scales, k, v, True)
    wide_ts = api.NVFP4Tensor(q.codes, q.scales, torch.zeros(2))
    with pytest.raises(ValueError, match="q.tensor_scale"):
        api.attn_qk4v8_fwd(wide_ts, k, v, True)
    as_int8 = api.NVFP4Tensor(q.codes.view(torch.int8), q.scales, q.tensor_scale)
    with pytest.raises(TypeError, match="q.codes"):
        api.attn_qk4v8_fwd(as_int8, k, v, True)
    with pytest.raises(ValueError, match="q.codes must be"):
        api.attn_qk4v8_fwd(api.NVFP4Tensor(q.codes[0], q.scales[0], q.tensor_scale), k, v, True)


def test_fwd_fp16_tiles_need_their_copies_and_a_full_bitmap():
    q16, k16 = _inputs16(1, 4, 2, 700, 700, 128)
    q, k, v = _prefill(1, 4, 2, 700, 700, 128)                      # no fp16 copy of V
    with pytest.raises(ValueError, match="want_fp16_v"):
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700), q16=q16, k16=k16)
    q, k, v = _prefill(1, 4, 2, 700, 700, 128, fp16=True)
    with pytest.raises(ValueError, match="q16 and k16"):
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700))
    with pytest.raises(TypeError, match="k16"):                       # Q and K of two types
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700), q16=q16, k16=k16.half())
    with pytest.raises(TypeError, match="q16"):
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700), q16=q16.float(), k16=k16)
    with pytest.raises(ValueError, match="k16"):                      # K of another length
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700), q16=q16, k16=k16[:, :, :600])
    with pytest.raises(ValueError, match="fp16_bitmap"):
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 2, 700), q16=q16, k16=k16)
    with pytest.raises(ValueError, match="second Q"):
        api.attn_qk4v8_fwd(q, k, v, True, fp16_bitmap=_bitmap(1, 4, 700), q2=q, q16=q16, k16=k16)


def test_strided_views_are_refused_before_any_call():
    q, k, v = _prefill(1, 4, 2, 256, 256, 128)
    # a transposed view with the right shape: the library would read it as dense
    tv = torch.empty(1, 2, 256 // 32, 128, dtype=torch.uint8).transpose(2, 3)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.attn_qk4v8_fwd(q, k, api.MXFP8V(v.codes, tv, 256), True)


def _decode(S=3, Hq=8, Hkv=2, D=128, pages=40, max_pages=16):
    q = api._nvfp4_empty((S, Hq, D), "cpu")
    cache = paged.empty_cache(pages, Hkv, D, 0.0625, "cpu")
    table = torch.full((S, max_pages), -1, dtype=torch.int32)
    ctx = torch.ones(S, dtype=torch.int32)
    return q, cache, table, ctx


@pytest.mark.parametrize("S,Hq,Hkv,D", [(3, 8, 2, 128), (64, 32, 8, 128), (5, 8, 2, 64), (1, 16, 1, 128)])
def test_decode_accepts_producer_shapes(S, Hq, Hkv, D):
    q, cache, table, ctx = _decode(S, Hq, Hkv, D)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.attn_qk4v8_decode_paged(q, cache, table, ctx, 1000, 256, want_lse=True,
                                    q2=api._nvfp4_empty((S, Hq, D), "cpu"))
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.attn_qk4v8_decode_paged_noalloc(q, cache, table, ctx, 1000, 256)
    out = torch.empty(S, Hq, D, dtype=torch.float32)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.decode_params(q, cache, table, ctx, 1 << 20, 128, out)


def test_decode_refuses_mismatched_buffers():
    q, cache, table, ctx = _decode()
    with pytest.raises(TypeError, match="page_table"):
        api.attn_qk4v8_decode_paged(q, cache, table.long(), ctx, 1000, 256)
    with pytest.raises(ValueError, match="context_lens"):
        api.attn_qk4v8_decode_paged(q, cache, table, ctx[:2].contiguous(), 1000, 256)
    with pytest.raises(ValueError, match="page_table"):
        api.attn_qk4v8_decode_paged(q, cache, table[:2].contiguous(), ctx, 1000, 256)
    one_v_head = paged.empty_cache(40, 2, 128, 0.0625, "cpu")
    one_v_head.v_pages = one_v_head.v_pages[:, :1].contiguous()     # V pages of one KV head
    with pytest.raises(ValueError, match="cache.v_pages"):
        api.attn_qk4v8_decode_paged(q, one_v_head, table, ctx, 1000, 256)
    with pytest.raises(ValueError, match="q2.codes"):
        api.attn_qk4v8_decode_paged(q, cache, table, ctx, 1000, 256,
                                    q2=api._nvfp4_empty((3, 4, 128), "cpu"))


def _append(S=4, Hkv=3, D=128, total=100, dtype=torch.bfloat16, pages=40, max_pages=8):
    cache = paged.empty_cache(pages, Hkv, D, 0.0625, "cpu")
    k = torch.empty(total, Hkv, D, dtype=dtype)
    cu = torch.zeros(S + 1, dtype=torch.int32)
    lens = torch.zeros(S, dtype=torch.int32)
    table = torch.zeros(S, max_pages, dtype=torch.int32)
    tail = paged.empty_tail(S, Hkv, D, dtype, "cpu")
    return cache, k, k.clone(), cu, lens, table, tail


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_append_accepts_producer_shapes(dtype):
    args = _append(dtype=dtype)
    with pytest.raises(ValueError, match=DEVICE_ERR):
        api.kv_append_paged(*args, max_new=100)


def test_append_refuses_mismatched_buffers():
    cache, k, v, cu, lens, table, tail = _append()
    with pytest.raises(ValueError, match="cu_new"):
        api.kv_append_paged(cache, k, v, cu[:-1].contiguous(), lens, table, tail, max_new=1)
    with pytest.raises(ValueError, match="v_tail"):
        api.kv_append_paged(cache, k, v, cu, lens, table, tail[:, :2].contiguous(), max_new=1)
    with pytest.raises(ValueError, match="share a dtype"):
        api.kv_append_paged(cache, k, v.half(), cu, lens, table, tail, max_new=1)
    with pytest.raises(ValueError, match="v_new"):
        api.kv_append_paged(cache, k, v[:50].contiguous(), cu, lens, table, tail, max_new=1)
    with pytest.raises(ValueError, match="cache.k_pages"):
        api.kv_append_paged(paged.empty_cache(40, 3, 64, 0.0625, "cpu"), k, v, cu, lens, table,
                            tail, max_new=1)


def test_dual_q_with_fp16_tiles_is_refused_before_any_work():
    x = torch.zeros(1, 2, 128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="dual_q"):
        api.qk4v8_attention(x, x, x, True, fp16_frac_bp=500, dual_q=True)
