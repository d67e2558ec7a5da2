"""Torch-facing binding of libqk4v8.so: the C entry points under the same names.

These functions allocate outputs and workspaces with torch on the input's device, take the
current CUDA stream, and pass raw pointers to the library. They do no arithmetic of their own:
every step of the path runs in the library's kernels, and a missing library raises.
"""
from __future__ import annotations

import ctypes as C
import math
from dataclasses import dataclass

import torch

from . import _lib

_DT = {torch.float16: _lib.QK4V8_F16, torch.bfloat16: _lib.QK4V8_BF16}
_OUT_DT = {**_DT, torch.float32: _lib.QK4V8_F32}


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"expected fp16 or bf16, got {t.dtype}")
    return _DT[t.dtype]


# The library derives every buffer's extent from the sizes it is given and takes plain device
# pointers, so a host tensor, a strided view or a buffer of the wrong shape would be read (or
# written) as if it had the dense layout those sizes imply. These checks run before any call.
def _expect(t, name: str, shape, dtype) -> None:
    if t is None:
        raise ValueError(f"{name} is required")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")


def _expect_dims(t, name: str, ndim: int, layout: str) -> None:
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {layout}, got shape {tuple(t.shape)}")


def _expect_scalar(t, name: str) -> None:
    if t is None or t.numel() != 1 or t.dtype != torch.float32:
        raise ValueError(f"{name} must be a one-element float32 tensor")


def _on_one_gpu(*ts) -> None:
    ts = [t for t in ts if t is not None]
    dev = ts[0].get_device()
    for t in ts:
        if not t.is_cuda or t.get_device() != dev or not t.is_contiguous():
            raise ValueError("the library takes contiguous tensors on one CUDA device")


def _nvfp4_empty(shape, device, want_fp16: bool = False) -> NVFP4Tensor:
    """Uninitialised NVFP4 output for an input of ``shape`` (..., D)."""
    lead, cols = tuple(shape[:-1]), shape[-1]
    return NVFP4Tensor(torch.empty(*lead, cols // 2, dtype=torch.uint8, device=device),
                       torch.empty(*lead, cols // 16, dtype=torch.uint8, device=device),
                       torch.empty(1, dtype=torch.float32, device=device),
                       torch.empty(tuple(shape), dtype=torch.float16, device=device) if want_fp16 else None)


def _mxfp8_empty(shape, device, want_fp16: bool = False) -> MXFP8V:
    """Uninitialised MXFP8 output for V of ``shape`` (..., N, D): [..., D, N_pad128]."""
    lead, n, d = tuple(shape[:-2]), shape[-2], shape[-1]
    npad = (n + 127) // 128 * 128
    return MXFP8V(torch.empty(*lead, d, npad, dtype=torch.uint8, device=device),
                  torch.empty(*lead, d, npad // 32, dtype=torch.uint8, device=device), n,
                  torch.empty(*lead, d, npad, dtype=torch.float16, device=device) if want_fp16 else None)


@dataclass
class NVFP4Tensor:
    """NVFP4 codes [..., D/2], E4M3 scales [..., D/16], FP32 tensor scale (1-element device
    tensor) and, on request, an fp16 copy of the input [..., D]."""
    codes: torch.Tensor
    scales: torch.Tensor
    tensor_scale: torch.Tensor
    fp16: torch.Tensor | None = None


@dataclass
class MXFP8V:
    """MXFP8 V: codes [..., D, Npad] (token-contiguous), E8M0 scales [..., D, Npad/32], the
    true token count, and on request an fp16 copy [..., D, Npad]."""
    codes: torch.Tensor
    scales: torch.Tensor
    n_tokens: int
    fp16: torch.Tensor | None = None


def check_status(stream=None) -> int:
    """Synchronise the stream and return the device status (0 = ok); see qk4v8_check_status."""
    s = C.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    return _lib.load().qk4v8_check_status(s)


def timeout_site() -> dict | None:
    """Decode qk4v8_timeout_site(): where the first timed-out device wait sat, or None."""
    v = _lib.load().qk4v8_timeout_site()
    if v == 0:
        return None
    return {"kernel": {1: "attn_fwd", 2: "decode", 3: "selftest"}.get(v >> 56, v >> 56),
            "role": {0: "producer", 1: "mma", 2: "softmax"}.get((v >> 48) & 0xFF, (v >> 48) & 0xFF),
            "barrier": (v >> 40) & 0xFF, "tile": (v >> 20) & 0xFFFFF, "block": v & 0xFFFFF}


def selftest_wait_timeout() -> None:
    """Launch the bounded-wait self-test kernel (times out after about a second)."""
    _lib.check(_lib.load().qk4v8_selftest_wait_timeout(_stream()), "qk4v8_selftest_wait_timeout")


def quantize_nvfp4(x: torch.Tensor, tensor_scale: float | None = None, want_fp16: bool = False,
                   workspace: torch.Tensor | None = None, scale_search: bool = False,
                   out: NVFP4Tensor | None = None) -> NVFP4Tensor:
    """NVFP4-quantize ``x`` (..., D) along its last axis (contiguous fp16/bf16 CUDA tensor).

    ``tensor_scale``: a fixed FP32 tensor scale (a paged cache's, for instance); None or a
    value <= 0 computes it from the tensor's amax (amax / (6 * 448)). ``want_fp16`` also
    writes an fp16 copy of ``x`` for the FP16-tile attention path. ``workspace``: optional
    uint8 scratch of ``quantize_nvfp4_workspace_size()`` bytes. ``scale_search`` picks each
    block's scale among four candidates by squared error. ``out``: optional preallocated
    result (from a previous call on the same shape), written in place instead of allocating."""
    lib = _lib.load()
    if not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous CUDA tensor")
    cols = x.shape[-1]
    rows = x.numel() // cols
    if out is None:
        r = _nvfp4_empty(x.shape, x.device, want_fp16)
    else:
        r = out
        lead = tuple(x.shape[:-1])
        _expect(r.codes, "out.codes", lead + (cols // 2,), torch.uint8)
        _expect(r.scales, "out.scales", lead + (cols // 16,), torch.uint8)
        _expect_scalar(r.tensor_scale, "out.tensor_scale")
        if want_fp16:
            _expect(r.fp16, "out.fp16", tuple(x.shape), torch.float16)
        _on_one_gpu(x, r.codes, r.scales, r.tensor_scale, r.fp16 if want_fp16 else None)
    need = lib.quantize_nvfp4_workspace_size()
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    elif workspace.numel() < need or workspace.dtype != torch.uint8:
        raise ValueError(f"workspace must hold {need} bytes (uint8)")
    _on_one_gpu(x, workspace)
    fn = lib.quantize_nvfp4_searched if scale_search else lib.quantize_nvfp4
    st = fn(_ptr(x), _dtype(x), rows, cols, cols,
            float(tensor_scale) if tensor_scale else 0.0, _ptr(r.codes), _ptr(r.scales),
            _ptr(r.tensor_scale), _ptr(r.fp16) if want_fp16 else None, _ptr(workspace),
            workspace.numel(), _stream())
    _lib.check(st, "quantize_nvfp4")
    return r


def qk_smooth_rotate(x: torch.Tensor, role: str, lam: torch.Tensor | None = None) -> torch.Tensor:
    """Outlier-aware transform of queries (role 'q': x * lam) or keys ('k': x / lam) along the
    last axis (128): per-channel smoothing, the 128-point Hadamard rotation and 2^-3 / 2^-4,
    so that transformed queries and keys keep their dot products. Returns a new tensor."""
    if not x.is_cuda or not x.is_contiguous() or x.shape[-1] != 128:
        raise ValueError("x must be a contiguous CUDA tensor with last dimension 128")
    if lam is not None and (lam.dtype != torch.float32 or lam.numel() != 128):
        raise ValueError("lam must be 128 float32 values")
    _on_one_gpu(x, lam)
    out = torch.empty_like(x)
    st = _lib.load().qk_smooth_rotate(_ptr(x), _dtype(x), x.numel() // 128, 128, _ptr(lam),
                                      0 if role == "q" else 1, _ptr(out), _stream())
    _lib.check(st, "qk_smooth_rotate")
    return out


def quantize_nvfp4_dual(x: torch.Tensor, tensor_scale: float | None = None):
    """Dual-residual NVFP4: (Q1, Q2) with Q1 = quantize_nvfp4(x) and Q2 the encoding of
    x - Q1's values under Q1's tensor scale (shared tensor-scale tensor)."""
    q1 = quantize_nvfp4(x, tensor_scale)             # checks x
    cols = x.shape[-1]
    codes2, scales2 = torch.empty_like(q1.codes), torch.empty_like(q1.scales)
    st = _lib.load().quantize_nvfp4_residual(_ptr(x), _dtype(x), x.numel() // cols, cols, cols,
                                             _ptr(q1.codes), _ptr(q1.scales),
                                             _ptr(q1.tensor_scale), _ptr(codes2), _ptr(scales2),
                                             _stream())
    _lib.check(st, "quantize_nvfp4_residual")
    return q1, NVFP4Tensor(codes2, scales2, q1.tensor_scale)


def quantize_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, want_fp16_v: bool = False,
                 workspace: torch.Tensor | None = None):
    """Q and K (..., D) to NVFP4 with their own tensor scales and V (..., N, D) to MXFP8, in two
    launches (quantize_qkv); the same outputs as quantize_nvfp4(q), quantize_nvfp4(k) and
    quantize_mxfp8_v(v). ``want_fp16_v`` also writes V's fp16 copy (v8.fp16), the one 16-bit
    operand the FP16-tile attention needs besides the caller's Q and K. Returns (q4, k4, v8)."""
    lib = _lib.load()
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if not (q.dtype == k.dtype == v.dtype):
        raise TypeError("q, k and v must share a dtype")
    d = q.shape[-1]
    if k.shape[-1] != d or v.shape[-1] != d or v.dim() < 2:
        raise ValueError("q, k and v must share the last (head) dimension; v is (..., N, D)")
    need = lib.quantize_qkv_workspace_size()
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    elif workspace.numel() < need or workspace.dtype != torch.uint8:
        raise ValueError(f"workspace must hold {need} bytes (uint8)")
    _on_one_gpu(q, k, v, workspace)
    q4 = _nvfp4_empty(q.shape, q.device)
    k4 = _nvfp4_empty(k.shape, k.device)
    v8 = _mxfp8_empty(v.shape, v.device, want_fp16_v)
    n = v.shape[-2]
    p = _lib.QkvParams(
        q=_ptr(q), k=_ptr(k), v=_ptr(v), dtype=_dtype(q), head_dim=d,
        q_rows=q.numel() // d, k_rows=k.numel() // d, v_bh=v.numel() // (n * d), v_tokens=n,
        q_codes=_ptr(q4.codes), q_scales=_ptr(q4.scales), q_tensor_scale=_ptr(q4.tensor_scale),
        k_codes=_ptr(k4.codes), k_scales=_ptr(k4.scales), k_tensor_scale=_ptr(k4.tensor_scale),
        v_codes=_ptr(v8.codes), v_scales=_ptr(v8.scales), q16=None, k16=None, v16=_ptr(v8.fp16))
    _lib.check(lib.quantize_qkv(C.byref(p), _ptr(workspace), workspace.numel(), _stream()),
               "quantize_qkv")
    return q4, k4, v8


def quantize_mxfp8_v(v: torch.Tensor, want_fp16: bool = False) -> MXFP8V:
    """MXFP8-quantize V laid out (..., N, D) along the token axis."""
    lib = _lib.load()
    if not v.is_cuda or not v.is_contiguous():
        raise ValueError("v must be a contiguous CUDA tensor")
    n, d = v.shape[-2], v.shape[-1]
    bh = v.numel() // (n * d)
    r = _mxfp8_empty(v.shape, v.device, want_fp16)
    st = lib.quantize_mxfp8_v(_ptr(v), _dtype(v), bh, n, d, _ptr(r.codes), _ptr(r.scales),
                              _ptr(r.fp16), _stream())
    _lib.check(st, "quantize_mxfp8_v")
    return r


def tile_score_select(q: NVFP4Tensor, k: NVFP4Tensor, causal: bool, frac_bp: int,
                      k_max: int | None = None):
    """Top-fraction tile selection. q.codes [B, Hq, N, D/2], k.codes [B, Hkv, N, D/2].
    Returns (idx [B*Hq, k_max] rank-ordered, n_sel [B*Hq], bitmap [B*Hq, T, T])."""
    _expect_dims(q.codes, "q.codes", 4, "[B, Hq, N, D/2]")
    _expect_dims(k.codes, "k.codes", 4, "[B, Hkv, N, D/2]")
    B, Hq, N, dh = q.codes.shape
    Hkv = k.codes.shape[1]
    d = dh * 2
    _expect(q.codes, "q.codes", (B, Hq, N, d // 2), torch.uint8)
    _expect(q.scales, "q.scales", (B, Hq, N, d // 16), torch.uint8)
    _expect(k.codes, "k.codes", (B, Hkv, N, d // 2), torch.uint8)
    _expect(k.scales, "k.scales", (B, Hkv, N, d // 16), torch.uint8)
    _on_one_gpu(q.codes, q.scales, k.codes, k.scales)
    lib = _lib.load()
    T = (N + 127) // 128
    n_cand = T * (T + 1) // 2 if causal else T * T
    need = (n_cand * frac_bp + 9999) // 10000
    k_max = max(need, 1) if k_max is None else k_max
    dev = q.codes.device
    idx = torch.full((B * Hq, k_max), -1, dtype=torch.int32, device=dev)
    n_sel = torch.empty(B * Hq, dtype=torch.int32, device=dev)
    bitmap = torch.empty(B * Hq, T, T, dtype=torch.uint8, device=dev)
    wsb = lib.tile_score_select_workspace_size(B, Hq, Hkv, N)
    ws = torch.empty(max(wsb, 8), dtype=torch.uint8, device=dev)
    st = lib.tile_score_select(_ptr(q.codes), _ptr(q.scales), _ptr(k.codes), _ptr(k.scales),
                               B, Hq, Hkv, N, d, int(causal), int(frac_bp), int(k_max),
                               _ptr(idx), _ptr(n_sel), _ptr(bitmap), _ptr(ws), ws.numel(),
                               _stream())
    _lib.check(st, "tile_score_select")
    return idx, n_sel, bitmap


def attn_qk4v8_fwd(q: NVFP4Tensor, k: NVFP4Tensor, v: MXFP8V, causal: bool,
                   softmax_scale: float | None = None, out_dtype=torch.bfloat16,
                   fp16_bitmap: torch.Tensor | None = None, want_lse: bool = False,
                   underflow_aware: bool = False, q2: NVFP4Tensor | None = None,
                   q16: torch.Tensor | None = None, k16: torch.Tensor | None = None):
    """QK4V8 attention forward. q.codes [B, Hq, Nq, D/2], k.codes [B, Hkv, Nk, D/2],
    v.codes [B, Hkv, D, Nk_pad]. With ``fp16_bitmap`` the selected tiles read the 16-bit Q and
    K the codes were quantized from (``q16`` [B, Hq, Nq, D], ``k16`` [B, Hkv, Nk, D], fp16 or
    bf16, one type) and V's fp16 copy (v.fp16, from quantize_qkv(want_fp16_v=True)).
    Returns out [B, Hq, Nq, D] (and lse [B, Hq, Nq])."""
    _expect_dims(q.codes, "q.codes", 4, "[B, Hq, Nq, D/2]")
    _expect_dims(k.codes, "k.codes", 4, "[B, Hkv, Nk, D/2]")
    B, Hq, Nq, dh = q.codes.shape
    Hkv, Nk = k.codes.shape[1], k.codes.shape[2]
    d = dh * 2
    npad = (Nk + 127) // 128 * 128
    _expect(q.codes, "q.codes", (B, Hq, Nq, d // 2), torch.uint8)
    _expect(q.scales, "q.scales", (B, Hq, Nq, d // 16), torch.uint8)
    _expect_scalar(q.tensor_scale, "q.tensor_scale")
    _expect(k.codes, "k.codes", (B, Hkv, Nk, d // 2), torch.uint8)
    _expect(k.scales, "k.scales", (B, Hkv, Nk, d // 16), torch.uint8)
    _expect_scalar(k.tensor_scale, "k.tensor_scale")
    _expect(v.codes, "v.codes", (B, Hkv, d, npad), torch.uint8)
    _expect(v.scales, "v.scales", (B, Hkv, d, npad // 32), torch.uint8)
    bufs = [q.codes, q.scales, q.tensor_scale, k.codes, k.scales, k.tensor_scale, v.codes, v.scales]
    if fp16_bitmap is not None:
        if q2 is not None:
            raise ValueError("the second Q tensor is not combined with FP16 tiles")
        tiles = B * Hq * ((Nq + 127) // 128) * ((Nk + 127) // 128)
        if fp16_bitmap.dtype != torch.uint8 or fp16_bitmap.numel() != tiles:
            raise ValueError(f"fp16_bitmap must hold {tiles} uint8 tile flags")
        if q16 is None or k16 is None:
            raise ValueError("FP16 tiles need q16 and k16 (the 16-bit Q and K)")
        if q16.dtype not in (torch.float16, torch.bfloat16):
            raise TypeError(f"q16: dtype {q16.dtype}, expected float16 or bfloat16")
        _expect(q16, "q16", (B, Hq, Nq, d), q16.dtype)
        _expect(k16, "k16", (B, Hkv, Nk, d), q16.dtype)
        _expect(v.fp16, "v.fp16 (quantize with want_fp16_v=True)", (B, Hkv, d, npad), torch.float16)
        bufs += [fp16_bitmap, q16, k16, v.fp16]
    if q2 is not None:
        _expect(q2.codes, "q2.codes", (B, Hq, Nq, d // 2), torch.uint8)
        _expect(q2.scales, "q2.scales", (B, Hq, Nq, d // 16), torch.uint8)
        bufs += [q2.codes, q2.scales]
    _on_one_gpu(*bufs)
    lib = _lib.load()
    out = torch.empty(B, Hq, Nq, d, dtype=out_dtype, device=q.codes.device)
    lse = torch.empty(B, Hq, Nq, dtype=torch.float32, device=q.codes.device) if want_lse else None
    p = _lib.FwdParams()
    p.q_codes, p.q_scales, p.q_tensor_scale = q.codes.data_ptr(), q.scales.data_ptr(), q.tensor_scale.data_ptr()
    p.k_codes, p.k_scales, p.k_tensor_scale = k.codes.data_ptr(), k.scales.data_ptr(), k.tensor_scale.data_ptr()
    p.v_codes, p.v_scales = v.codes.data_ptr(), v.scales.data_ptr()
    p.batch, p.q_heads, p.kv_heads, p.n_q, p.n_k, p.head_dim = B, Hq, Hkv, Nq, Nk, d
    p.causal = int(causal)
    p.softmax_scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    if fp16_bitmap is not None:
        p.fp16_bitmap = fp16_bitmap.data_ptr()
        p.q16, p.k16, p.v16 = q16.data_ptr(), k16.data_ptr(), v.fp16.data_ptr()
        p.qk16_dtype = _dtype(q16)
    p.out_dtype = _OUT_DT[out_dtype]
    p.out = out.data_ptr()
    p.lse = lse.data_ptr() if lse is not None else None
    p.p_underflow_aware = int(bool(underflow_aware))
    if q2 is not None:                      # dual-residual Q: S = (Q1 + Q2) K^T
        p.q2_codes, p.q2_scales = q2.codes.data_ptr(), q2.scales.data_ptr()
    _lib.check(lib.attn_qk4v8_fwd(C.byref(p), _stream()), "attn_qk4v8_fwd")
    return (out, lse) if want_lse else out


@dataclass
class PagedKV:
    """Paged NVFP4-K / MXFP8-V cache (64-token pages)."""
    k_pages: torch.Tensor        # [P, Hkv, 64, D/2]
    k_scales: torch.Tensor       # [P, Hkv, 64, D/16]
    k_tensor_scale: torch.Tensor  # [1] float
    v_pages: torch.Tensor        # [P, Hkv, D, 64]
    v_scales: torch.Tensor       # [P, Hkv, D, 2]


def decode_params(q: NVFP4Tensor, cache: PagedKV, page_table: torch.Tensor,
                  context_lens: torch.Tensor, max_context: int, split_tokens: int,
                  out: torch.Tensor, softmax_scale: float | None = None, lse=None,
                  underflow_aware: bool = False, q2: NVFP4Tensor | None = None):
    """The decode parameter struct, after checking every buffer against the sizes it states."""
    _expect_dims(q.codes, "q.codes", 3, "[S, Hq, D/2]")
    _expect_dims(cache.k_pages, "cache.k_pages", 4, "[P, Hkv, 64, D/2]")
    _expect_dims(page_table, "page_table", 2, "[S, max_pages]")
    S, Hq, dh = q.codes.shape
    P, Hkv = cache.k_pages.shape[0], cache.k_pages.shape[1]
    d = dh * 2
    _expect(q.scales, "q.scales", (S, Hq, d // 16), torch.uint8)
    _expect_scalar(q.tensor_scale, "q.tensor_scale")
    _expect(cache.k_pages, "cache.k_pages", (P, Hkv, 64, d // 2), torch.uint8)
    _expect(cache.k_scales, "cache.k_scales", (P, Hkv, 64, d // 16), torch.uint8)
    _expect_scalar(cache.k_tensor_scale, "cache.k_tensor_scale")
    _expect(cache.v_pages, "cache.v_pages", (P, Hkv, d, 64), torch.uint8)
    _expect(cache.v_scales, "cache.v_scales", (P, Hkv, d, 2), torch.uint8)
    _expect(page_table, "page_table", (S, page_table.shape[1]), torch.int32)
    _expect(context_lens, "context_lens", (S,), torch.int32)
    _expect(out, "out", (S, Hq, d), out.dtype)
    bufs = [q.codes, q.scales, q.tensor_scale, cache.k_pages, cache.k_scales, cache.k_tensor_scale,
            cache.v_pages, cache.v_scales, page_table, context_lens, out]
    if lse is not None:
        _expect(lse, "lse", (S, Hq), torch.float32)
        bufs.append(lse)
    if q2 is not None:
        _expect(q2.codes, "q2.codes", (S, Hq, d // 2), torch.uint8)
        _expect(q2.scales, "q2.scales", (S, Hq, d // 16), torch.uint8)
        bufs += [q2.codes, q2.scales]
    _on_one_gpu(*bufs)
    p = _lib.DecodeParams()
    p.q_codes, p.q_scales, p.q_tensor_scale = q.codes.data_ptr(), q.scales.data_ptr(), q.tensor_scale.data_ptr()
    p.k_pages, p.k_page_scales, p.k_tensor_scale = (cache.k_pages.data_ptr(), cache.k_scales.data_ptr(),
                                                    cache.k_tensor_scale.data_ptr())
    p.v_pages, p.v_page_scales = cache.v_pages.data_ptr(), cache.v_scales.data_ptr()
    p.page_table, p.context_lens = page_table.data_ptr(), context_lens.data_ptr()
    p.num_seqs, p.num_pages, p.max_pages = S, P, page_table.shape[1]
    p.q_heads, p.kv_heads, p.head_dim = Hq, Hkv, d
    p.max_context, p.split_tokens = int(max_context), int(split_tokens)
    p.softmax_scale = 1.0 / math.sqrt(d) if softmax_scale is None else softmax_scale
    p.out_dtype = _OUT_DT[out.dtype]
    p.out = out.data_ptr()
    p.lse = lse.data_ptr() if lse is not None else None
    p.p_underflow_aware = int(bool(underflow_aware))
    if q2 is not None:                      # dual-residual Q
        p.q2_codes, p.q2_scales = q2.codes.data_ptr(), q2.scales.data_ptr()
    return p


def attn_qk4v8_decode_paged(q: NVFP4Tensor, cache: PagedKV, page_table: torch.Tensor,
                            context_lens: torch.Tensor, max_context: int, split_tokens: int,
                            softmax_scale: float | None = None, out_dtype=torch.bfloat16,
                            want_lse: bool = False, workspace: torch.Tensor | None = None,
                            underflow_aware: bool = False, q2: NVFP4Tensor | None = None):
    """One decode step. q.codes [S, Hq, D/2]; returns out [S, Hq, D] (and lse [S, Hq]).
    ``underflow_aware`` scales P per 32-key block by a power of two before its E4M3 encode."""
    S, Hq, dh = q.codes.shape
    out = torch.empty(S, Hq, dh * 2, dtype=out_dtype, device=q.codes.device)
    lse = torch.empty(S, Hq, dtype=torch.float32, device=q.codes.device) if want_lse else None
    p = decode_params(q, cache, page_table, context_lens, max_context, split_tokens, out,
                      softmax_scale, lse, underflow_aware, q2)
    lib = _lib.load()
    need = lib.attn_qk4v8_decode_workspace_size(C.byref(p))
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.codes.device)
    elif workspace.dtype != torch.uint8:
        raise TypeError("workspace must be a uint8 tensor")
    else:
        _on_one_gpu(q.codes, workspace)
    st = lib.attn_qk4v8_decode_paged(C.byref(p), _ptr(workspace), workspace.numel(), _stream())
    _lib.check(st, "attn_qk4v8_decode_paged")
    return (out, lse) if want_lse else out


class DecodePlan:
    """A decode step whose fixed buffers are checked once: the paged cache, page table,
    context lengths, split, output (and lse) buffers and workspace. ``run(q)`` then checks only
    the step's query and launches through attn_qk4v8_decode_paged, writing into the plan's own
    output buffer (read it before the next ``run``). For serving loops, where the per-step
    host work of checking and allocating would otherwise show up between the launches."""

    def __init__(self, cache: PagedKV, page_table: torch.Tensor, context_lens: torch.Tensor,
                 max_context: int, split_tokens: int, num_seqs: int, q_heads: int,
                 softmax_scale: float | None = None, out_dtype=torch.bfloat16,
                 want_lse: bool = False, workspace: torch.Tensor | None = None,
                 underflow_aware: bool = False):
        d = cache.k_pages.shape[-1] * 2
        dev = cache.k_pages.device
        self.q_shape = (num_seqs, q_heads, d // 2)
        self.out = torch.empty(num_seqs, q_heads, d, dtype=out_dtype, device=dev)
        self.lse = torch.empty(num_seqs, q_heads, dtype=torch.float32, device=dev) if want_lse else None
        # a stand-in query of the step's shape: checks every fixed buffer against it once
        probe = NVFP4Tensor(torch.empty(self.q_shape, dtype=torch.uint8, device=dev),
                            torch.empty(num_seqs, q_heads, d // 16, dtype=torch.uint8, device=dev),
                            torch.empty(1, dtype=torch.float32, device=dev))
        self.params = decode_params(probe, cache, page_table, context_lens, max_context,
                                    split_tokens, self.out, softmax_scale, self.lse,
                                    underflow_aware)
        self._keep = (cache, page_table, context_lens)
        lib = _lib.load()
        need = lib.attn_qk4v8_decode_workspace_size(C.byref(self.params))
        if workspace is None or workspace.numel() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        elif workspace.dtype != torch.uint8:
            raise TypeError("workspace must be a uint8 tensor")
        _on_one_gpu(self.out, workspace)
        self.workspace = workspace
        self._dev = dev.index if dev.index is not None else torch.cuda.current_device()

    def run(self, q: NVFP4Tensor):
        """One decode step for the quantized query ``q`` [S, Hq, D/2]; returns the plan's out
        (and lse)."""
        c, sc, ts = q.codes, q.scales, q.tensor_scale
        if tuple(c.shape) != self.q_shape or c.dtype != torch.uint8 or not c.is_cuda or \
                c.get_device() != self._dev or not c.is_contiguous() or not sc.is_contiguous() or \
                sc.get_device() != self._dev or ts.get_device() != self._dev or \
                sc.numel() * 8 != c.numel():
            raise ValueError(f"q must be an NVFP4 query of shape {self.q_shape} on the plan's device")
        p = self.params
        p.q_codes, p.q_scales, p.q_tensor_scale = c.data_ptr(), sc.data_ptr(), ts.data_ptr()
        st = _lib.load().attn_qk4v8_decode_paged(C.byref(p), _ptr(self.workspace),
                                                 self.workspace.numel(), _stream())
        _lib.check(st, "attn_qk4v8_decode_paged")
        return (self.out, self.lse) if self.lse is not None else self.out


def attn_qk4v8_decode_paged_noalloc(q: NVFP4Tensor, cache: PagedKV, page_table: torch.Tensor,
                                    context_lens: torch.Tensor, max_context: int,
                                    split_tokens: int, softmax_scale: float | None = None,
                                    out_dtype=torch.bfloat16, want_lse: bool = False):
    """The decode step through the library's allocation-free entry point: the library keeps
    the split partials in its own fixed 16 MiB device buffer instead of a caller workspace,
    for callers that cannot provide device memory. Only the output (and lse) are allocated
    here, as for every other entry point of this binding."""
    S, Hq, dh = q.codes.shape
    out = torch.empty(S, Hq, dh * 2, dtype=out_dtype, device=q.codes.device)
    lse = torch.empty(S, Hq, dtype=torch.float32, device=q.codes.device) if want_lse else None
    p = decode_params(q, cache, page_table, context_lens, max_context, split_tokens, out,
                      softmax_scale, lse)
    lib = _lib.load()
    st = lib.attn_qk4v8_decode_paged_noalloc(C.byref(p), _stream())
    _lib.check(st, "attn_qk4v8_decode_paged_noalloc")
    return (out, lse) if want_lse else out


def kv_append_paged(cache: PagedKV, k_new: torch.Tensor, v_new: torch.Tensor,
                    cu_new: torch.Tensor, lens: torch.Tensor, page_table: torch.Tensor,
                    v_tail: torch.Tensor, max_new: int) -> None:
    """Quantize new tokens into the paged cache in place. k_new, v_new [total_new, Hkv, D]
    (fp16/bf16); cu_new [S + 1] int32 offsets of each sequence's new rows; lens [S] int32
    lengths before the call (the caller adds the new counts); page_table [S, max_pages];
    v_tail [S, Hkv, D, 32] of k_new's dtype, each sequence's incomplete V group, updated."""
    _expect_dims(k_new, "k_new", 3, "[total_new, Hkv, D]")
    _expect_dims(cache.k_pages, "cache.k_pages", 4, "[P, Hkv, 64, D/2]")
    _expect_dims(page_table, "page_table", 2, "[S, max_pages]")
    if v_new.dtype != k_new.dtype or v_tail.dtype != k_new.dtype:
        raise ValueError("k_new, v_new and v_tail must share a dtype")
    _, hkv, d = k_new.shape
    S, P = lens.numel(), cache.k_pages.shape[0]
    _expect(v_new, "v_new", tuple(k_new.shape), k_new.dtype)
    _expect(cu_new, "cu_new", (S + 1,), torch.int32)
    _expect(lens, "lens", (S,), torch.int32)
    _expect(page_table, "page_table", (S, page_table.shape[1]), torch.int32)
    _expect(v_tail, "v_tail", (S, hkv, d, 32), k_new.dtype)
    _expect(cache.k_pages, "cache.k_pages", (P, hkv, 64, d // 2), torch.uint8)
    _expect(cache.k_scales, "cache.k_scales", (P, hkv, 64, d // 16), torch.uint8)
    _expect_scalar(cache.k_tensor_scale, "cache.k_tensor_scale")
    _expect(cache.v_pages, "cache.v_pages", (P, hkv, d, 64), torch.uint8)
    _expect(cache.v_scales, "cache.v_scales", (P, hkv, d, 2), torch.uint8)
    _on_one_gpu(k_new, v_new, cu_new, lens, page_table, v_tail, cache.k_pages, cache.k_scales,
                cache.k_tensor_scale, cache.v_pages, cache.v_scales)
    lib = _lib.load()
    p = _lib.AppendParams(
        k_new=_ptr(k_new), v_new=_ptr(v_new), dtype=_dtype(k_new), cu_new=_ptr(cu_new),
        lens=_ptr(lens), page_table=_ptr(page_table), k_pages=_ptr(cache.k_pages),
        k_page_scales=_ptr(cache.k_scales), k_tensor_scale=_ptr(cache.k_tensor_scale),
        v_pages=_ptr(cache.v_pages), v_page_scales=_ptr(cache.v_scales), v_tail=_ptr(v_tail),
        num_seqs=lens.numel(), num_pages=cache.k_pages.shape[0], max_pages=page_table.shape[1],
        kv_heads=hkv, head_dim=d, max_new=int(max_new))
    st = lib.kv_append_paged(C.byref(p), _stream())
    _lib.check(st, "kv_append_paged")


def qk4v8_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool,
                    softmax_scale: float | None = None, fp16_frac_bp: int = 0,
                    out_dtype=None, want_lse: bool = False, underflow_aware: bool = False,
                    dual_q: bool = False):
    """The whole prefill path on bf16/fp16 CUDA tensors q [B, Hq, N, D], k/v [B, Hkv, N, D]:
    quantize Q, K (NVFP4) and V (MXFP8), optionally score tiles and recompute the top
    ``fp16_frac_bp`` basis points of them in FP16, then attention. ``dual_q`` adds the
    residual second Q tensor; ``underflow_aware`` scales P per 32-key block."""
    mixed = fp16_frac_bp > 0
    if mixed and dual_q:
        raise ValueError("dual_q is not combined with FP16 tiles")
    q2 = None
    if dual_q:
        q4, q2 = quantize_nvfp4_dual(q)
        k4 = quantize_nvfp4(k)
        v8 = quantize_mxfp8_v(v)
    else:
        q4, k4, v8 = quantize_qkv(q, k, v, want_fp16_v=mixed)
    bitmap = None
    if mixed:
        _, _, bitmap = tile_score_select(q4, k4, causal, fp16_frac_bp)
    return attn_qk4v8_fwd(q4, k4, v8, causal, softmax_scale, out_dtype or q.dtype,
                          fp16_bitmap=bitmap, want_lse=want_lse, underflow_aware=underflow_aware,
                          q2=q2, q16=q if mixed else None, k16=k if mixed else None)
