"""Host-side checks of the C ABI (no GPU needed): the library loads, exports exactly what
include/qk4v8.h declares, its structs match the binding, and argument validation rejects bad
calls before touching the device."""
import ctypes as C
import os
import re

import pytest

from bit_block_scaled_nvfp4_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qk4v8.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)) -
                  {"if", "defined"})


def test_header_declares_the_bound_functions():
    names = declared_functions()
    assert set(names) == set(_lib.SIGNATURES), names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, flags=re.M), name


def test_struct_layouts_match(lib):
    assert lib.qk4v8_struct_size(0) == C.sizeof(_lib.FwdParams)
    assert lib.qk4v8_struct_size(1) == C.sizeof(_lib.DecodeParams)
    assert lib.qk4v8_struct_size(7) == 0


def test_version_and_status_strings(lib):
    assert lib.qk4v8_version() == 100
    assert lib.qk4v8_status_string(0) == b"ok"
    assert lib.qk4v8_status_string(4) == b"device wait timed out"
    assert lib.qk4v8_status_string(99) == b"unknown status"


FAKE = 1 << 20          # aligned fake device addresses: never dereferenced on these paths


def test_per_device_set_up_runs_once_per_device(lib):
    """The latch behind each kernel's shared-memory opt-in keeps one flag per device: the set-up
    step runs once for device 0 however often it is asked, and once more, on its own, for each
    other device; an out-of-range index is refused."""
    f = lib.qk4v8_selftest_device_once
    assert f(0) == 1 and f(0) == 1
    assert f(3) == 1 and f(3) == 1 and f(0) == 1
    assert f(63) == 1
    assert f(64) == -1 and f(-1) == -1


def test_quantize_nvfp4_validation(lib):
    f = lib.quantize_nvfp4
    ok = dict(x=FAKE, dt=1, rows=4, cols=64, stride=64, ts=0.0, codes=FAKE, scales=FAKE,
              tsout=FAKE, x16=None, ws=FAKE, wsb=4096)

    def call(**kw):
        a = dict(ok, **kw)
        return f(a["x"], a["dt"], a["rows"], a["cols"], a["stride"], a["ts"], a["codes"],
                 a["scales"], a["tsout"], a["x16"], a["ws"], a["wsb"], None)
    assert call(x=None) == _lib.QK4V8_ERR_INVALID_ARG
    assert call(cols=40) == _lib.QK4V8_ERR_INVALID_ARG            # not a multiple of 16
    assert call(stride=32) == _lib.QK4V8_ERR_INVALID_ARG          # stride < cols
    assert call(stride=68) == _lib.QK4V8_ERR_INVALID_ARG          # stride % 8
    assert call(x=FAKE + 2) == _lib.QK4V8_ERR_INVALID_ARG         # misaligned input
    assert call(ws=None) == _lib.QK4V8_ERR_INVALID_ARG            # amax pass needs workspace
    assert call(wsb=2) == _lib.QK4V8_ERR_INVALID_ARG
    assert call(dt=7) == _lib.QK4V8_ERR_INVALID_ARG


def test_quantize_qkv_validation(lib):
    """The fused Q/K/V quantize rejects bad calls on the host, before any launch."""
    assert lib.qk4v8_struct_size(3) == C.sizeof(_lib.QkvParams)
    f = lib.quantize_qkv
    wsb = lib.quantize_qkv_workspace_size()
    assert wsb >= 8

    def p(**kw):
        d = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, head_dim=128, q_rows=64, k_rows=16, v_bh=1,
                 v_tokens=16, q_codes=FAKE, q_scales=FAKE, q_tensor_scale=FAKE, k_codes=FAKE,
                 k_scales=FAKE, k_tensor_scale=FAKE, v_codes=FAKE, v_scales=FAKE)
        d.update(kw)
        return C.byref(_lib.QkvParams(**d))
    assert f(None, FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(p(v=None), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(p(k_tensor_scale=None), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(p(), None, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(p(), FAKE, wsb - 4, None) == _lib.QK4V8_ERR_INVALID_ARG     # short workspace
    assert f(p(dtype=2), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG   # fp32 input
    assert f(p(q_rows=0), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(p(head_dim=96), FAKE, wsb, None) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(p(q=FAKE + 8), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG   # misaligned
    assert f(p(q16=FAKE), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG     # Q, K copies: both or neither
    assert f(p(v16=FAKE + 8), FAKE, wsb, None) == _lib.QK4V8_ERR_INVALID_ARG # V copy misaligned


def test_quantize_mxfp8_validation(lib):
    f = lib.quantize_mxfp8_v
    assert f(None, 1, 1, 128, 128, FAKE, FAKE, None, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 0, 128, FAKE, FAKE, None, None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(FAKE, 1, 1, 128, 96, FAKE, FAKE, None, None) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(FAKE + 8, 1, 1, 128, 128, FAKE, FAKE, None, None) == _lib.QK4V8_ERR_INVALID_ARG


def test_tile_select_validation(lib):
    f = lib.tile_score_select
    args = [FAKE, FAKE, FAKE, FAKE, 1, 4, 2, 1000, 128, 1, 500, 64, FAKE, FAKE, None, FAKE, 1 << 20, None]
    bad_heads = list(args); bad_heads[5] = 3; bad_heads[6] = 2
    assert f(*bad_heads) == _lib.QK4V8_ERR_INVALID_ARG             # Hq % Hkv
    small_k = list(args); small_k[11] = 1
    assert f(*small_k) == _lib.QK4V8_ERR_INVALID_ARG               # k_max < ceil(36 * 5%) = 2
    big_k = list(args); big_k[11] = 5000
    assert f(*big_k) == _lib.QK4V8_ERR_UNSUPPORTED
    frac = list(args); frac[10] = 10001
    assert f(*frac) == _lib.QK4V8_ERR_INVALID_ARG
    ws = list(args); ws[16] = 8
    assert f(*ws) == _lib.QK4V8_ERR_INVALID_ARG


def _fwd(**kw):
    p = _lib.FwdParams()
    for n in ("q_codes", "q_scales", "q_tensor_scale", "k_codes", "k_scales", "k_tensor_scale",
              "v_codes", "v_scales", "out"):
        setattr(p, n, FAKE)
    p.batch, p.q_heads, p.kv_heads, p.n_q, p.n_k, p.head_dim = 1, 4, 2, 256, 256, 128
    p.causal, p.softmax_scale, p.out_dtype = 1, 0.125, 1
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_fwd_validation(lib):
    f = lambda p: lib.attn_qk4v8_fwd(C.byref(p), None)
    assert f(_fwd(q_codes=None)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_fwd(q_heads=3)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_fwd(n_k=300)) == _lib.QK4V8_ERR_INVALID_ARG        # causal needs Nq == Nk
    assert f(_fwd(head_dim=96)) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(_fwd(out=FAKE + 4)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_fwd(softmax_scale=0.0)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_fwd(fp16_bitmap=FAKE)) == _lib.QK4V8_ERR_INVALID_ARG  # bitmap without 16-bit operands
    assert f(_fwd(fp16_bitmap=FAKE, q16=FAKE, k16=FAKE, v16=FAKE, qk16_dtype=2)) == _lib.QK4V8_ERR_INVALID_ARG
    assert lib.attn_qk4v8_fwd(None, None) == _lib.QK4V8_ERR_INVALID_ARG


def _dec(**kw):
    p = _lib.DecodeParams()
    for n in ("q_codes", "q_scales", "q_tensor_scale", "k_pages", "k_page_scales",
              "k_tensor_scale", "v_pages", "v_page_scales", "page_table", "context_lens", "out"):
        setattr(p, n, FAKE)
    p.num_seqs, p.num_pages, p.max_pages = 2, 100, 50
    p.q_heads, p.kv_heads, p.head_dim = 32, 8, 128
    p.max_context, p.split_tokens, p.softmax_scale, p.out_dtype = 3000, 1024, 0.088, 1
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_decode_validation_and_workspace(lib):
    p = _dec()
    assert lib.attn_qk4v8_decode_workspace_size(C.byref(p)) == 2 * 32 * 3 * 130 * 4
    f = lambda p, wsb=1 << 30: lib.attn_qk4v8_decode_paged(C.byref(p), FAKE, wsb, None)
    assert f(_dec(split_tokens=100)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_dec(max_context=50 * 64 + 1)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_dec(head_dim=64)) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(_dec(q_heads=64, kv_heads=2)) == _lib.QK4V8_ERR_UNSUPPORTED  # g = 32 > 16
    assert f(_dec(), wsb=16) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_dec(page_table=None)) == _lib.QK4V8_ERR_INVALID_ARG
    # page rows beyond 32-bit tensor-map coordinates: refused before any map is built
    assert f(_dec(num_pages=(1 << 31) // (8 * 128))) == _lib.QK4V8_ERR_UNSUPPORTED


def _app(**kw):
    p = _lib.AppendParams(k_new=FAKE, v_new=FAKE, dtype=_lib.QK4V8_BF16, cu_new=FAKE, lens=FAKE,
                          page_table=FAKE, k_pages=FAKE, k_page_scales=FAKE, k_tensor_scale=FAKE,
                          v_pages=FAKE, v_page_scales=FAKE, v_tail=FAKE, num_seqs=4,
                          num_pages=64, max_pages=16, kv_heads=8, head_dim=128, max_new=32)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def test_append_validation(lib):
    f = lambda p: lib.kv_append_paged(C.byref(p), None)
    assert lib.qk4v8_struct_size(2) == C.sizeof(_lib.AppendParams)
    assert f(_app(v_tail=None)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(cu_new=None)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(dtype=_lib.QK4V8_F32)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(num_seqs=0)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(max_new=-1)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(head_dim=64)) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(_app(num_seqs=70000)) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(_app(k_new=FAKE + 8)) == _lib.QK4V8_ERR_INVALID_ARG    # not 16-byte aligned
    assert f(_app(v_pages=FAKE + 4)) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(_app(v_tail=FAKE + 2)) == _lib.QK4V8_ERR_INVALID_ARG


def test_quantize_residual_validation(lib):
    f = lambda **kw: lib.quantize_nvfp4_residual(*[dict(x=FAKE, dt=_lib.QK4V8_BF16, rows=4,
                                                        cols=64, stride=64, c=FAKE, s=FAKE,
                                                        ts=FAKE, c2=FAKE, s2=FAKE, st=None,
                                                        **{})[k] if k not in kw else kw[k]
                                                   for k in ("x", "dt", "rows", "cols", "stride",
                                                             "c", "s", "ts", "c2", "s2", "st")])
    assert f(x=None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(ts=None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(cols=40) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(c2=FAKE + 4) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(dt=_lib.QK4V8_F32) == _lib.QK4V8_ERR_INVALID_ARG


def test_smooth_rotate_validation(lib):
    f = lambda x=FAKE, dt=_lib.QK4V8_BF16, rows=4, hd=128, lam=None, role=0, out=FAKE: \
        lib.qk_smooth_rotate(x, dt, rows, hd, lam, role, out, None)
    assert f(x=None) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(role=2) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(hd=64) == _lib.QK4V8_ERR_UNSUPPORTED
    assert f(out=FAKE + 4) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(dt=_lib.QK4V8_F32) == _lib.QK4V8_ERR_INVALID_ARG
    assert f(rows=0) == _lib.QK4V8_OK                     # nothing to do, nothing launched


def test_product_path_fails_loudly_without_the_library(monkeypatch, tmp_path):
    """No CPU fallback: with the library absent every entry point raises instead of computing."""
    import torch
    from bit_block_scaled_nvfp4_b200 import api
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    monkeypatch.setattr(_lib, "_LIB", None)
    with pytest.raises(ImportError):
        _lib.load()
    with pytest.raises(ImportError):
        api.quantize_nvfp4(torch.zeros(4, 16, dtype=torch.bfloat16))
