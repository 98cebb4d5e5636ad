"""Host-only checks of the C ABI: the library loads, exports every function that
include/flexq.h declares, and rejects invalid arguments on the host (before any CUDA
call) with the documented status codes."""
import ctypes

import pytest

import group_wise_int4_b200 as fq


def test_library_exports_every_declared_function():
    L = fq.lib()
    names = fq.declared_functions()
    assert len(names) >= 16
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_binding_covers_every_declared_function():
    for n in fq.declared_functions():
        assert n in fq._SIGS, n
        assert hasattr(fq, n), n


def test_status_strings():
    assert fq.flex_status_string(0) == "ok"
    assert "timed out" in fq.flex_status_string(fq.FLEX_ERR_TIMEOUT)
    assert fq.flex_status_string(-99) == "unknown status"


def _shape(s):
    return fq._shape_arr(s)


def test_size_queries():
    L = fq.lib()
    cfg = fq.config(4, 64, 1)
    assert L.flexq_codes_bytes(2, _shape((4096, 4096)), cfg) == 4096 * 4096 // 2
    assert L.flexq_meta_bytes(2, _shape((4096, 4096)), cfg) == 4096 * 64 * 4
    assert L.flexq_codes_bytes(2, _shape((64, 96)), fq.config(8, 32, 0)) == 64 * 96
    assert L.flexq_meta_bytes(2, _shape((64, 96)), fq.config(8, 32, 0)) == 2 * 96 * 4
    # a partial last group is padded: ceil(100 / 64) = 2 groups per row
    assert L.flexq_codes_bytes(2, _shape((4, 100)), cfg) == 4 * 2 * 64 // 2
    assert L.flexq_meta_bytes(2, _shape((4, 100)), cfg) == 4 * 2 * 4
    # 3-bit codes: 3/8 byte per element; the symmetric form has the same sizes
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(3, 64, 1)) == 4 * 128 * 3 // 8
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(4, 64, 1, 1)) == 4 * 64
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(5, 64, 1)) == fq.FLEX_ERR_UNSUPPORTED
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(4, 48, 1)) == fq.FLEX_ERR_UNSUPPORTED
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(4, 64, 1, 2)) == fq.FLEX_ERR_UNSUPPORTED
    assert L.flexq_codes_bytes(5, _shape((4, 128)), cfg) == fq.FLEX_ERR_INVALID_ARG
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(4, 64, 2)) == fq.FLEX_ERR_INVALID_ARG
    # negative group_dim counts from the back
    assert L.flexq_codes_bytes(2, _shape((4, 128)), fq.config(4, 64, -1)) == 4 * 64


def test_codec_argument_errors_are_host_side():
    L = fq.lib()
    cfg = fq.config(4, 64, 1)
    shp = _shape((4, 128))
    P = ctypes.c_void_p
    assert L.flexq_compress(None, 2, shp, cfg, P(4096), P(8192), None) == fq.FLEX_ERR_INVALID_ARG
    assert L.flexq_compress(P(4096), 2, shp, cfg, P(4097), P(8192), None) == fq.FLEX_ERR_ALIGN
    assert L.flexq_compress(P(4104), 2, shp, cfg, P(4096), P(8192), None) == fq.FLEX_ERR_ALIGN
    assert L.flexq_decompress(P(4096), P(8192), 2, shp, cfg, P(4100), None) == fq.FLEX_ERR_ALIGN
    assert L.flexq_compress(P(4096), 2, _shape((4, 96)), fq.config(4, 64, 1, 3), P(4096), P(8192), None) == \
        fq.FLEX_ERR_UNSUPPORTED
    # an empty tensor is a valid no-op
    assert L.flexq_compress(P(4096), 2, _shape((0, 128)), cfg, P(4096), P(8192), None) == fq.FLEX_OK


def _cache_struct(**kw):
    c = fq.flex_kv_cache()
    c.k_codes, c.k_meta, c.v_codes, c.v_meta = 4096, 8192, 12288, 16384
    c.batch, c.n_heads, c.head_dim, c.max_seq = 2, 4, 64, 16
    c.cfg = fq.config(4, 64, 3)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_append_kv_argument_errors():
    L = fq.lib()
    P = ctypes.c_void_p
    ok = _cache_struct()
    assert L.flex_append_kv(ctypes.byref(ok), P(4096), P(8192), 256, 2, 16, None) == fq.FLEX_ERR_SHAPE
    assert L.flex_append_kv(ctypes.byref(ok), P(4096), P(8192), 256, 3, 0, None) == fq.FLEX_ERR_INVALID_ARG
    assert L.flex_append_kv(ctypes.byref(ok), P(4096), P(8192), 100, 2, 0, None) == fq.FLEX_ERR_INVALID_ARG
    assert L.flex_append_kv(ctypes.byref(ok), None, P(8192), 256, 2, 0, None) == fq.FLEX_ERR_INVALID_ARG
    assert L.flex_append_kv(ctypes.byref(ok), P(4098), P(8192), 256, 2, 0, None) == fq.FLEX_ERR_ALIGN
    bad = _cache_struct(head_dim=96)
    assert L.flex_append_kv(ctypes.byref(bad), P(4096), P(8192), 384, 2, 0, None) == fq.FLEX_ERR_UNSUPPORTED
    bad = _cache_struct(cfg=fq.config(4, 64, 3, 1))
    assert L.flex_append_kv(ctypes.byref(bad), P(4096), P(8192), 256, 2, 0, None) == fq.FLEX_ERR_UNSUPPORTED
    assert L.flex_append_kv(None, P(4096), P(8192), 256, 2, 0, None) == fq.FLEX_ERR_INVALID_ARG


def test_layernorm_argument_errors():
    L = fq.lib()
    P = ctypes.c_void_p
    assert L.flex_layernorm(None, P(16), P(32), P(48), 4, 64, None) == fq.FLEX_ERR_INVALID_ARG
    assert L.flex_layernorm(P(16), P(16), P(32), P(48), 4, 60, None) == fq.FLEX_ERR_UNSUPPORTED
    assert L.flex_layernorm(P(18), P(16), P(32), P(48), 4, 64, None) == fq.FLEX_ERR_ALIGN
    assert L.flex_layernorm(P(16), P(16), P(32), P(48), 0, 64, None) == fq.FLEX_OK


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(fq, "_lib", None)
    monkeypatch.setattr(fq, "LIB_PATH", str(tmp_path / "nope.so"))
    with pytest.raises(RuntimeError, match="missing"):
        fq.lib()


def test_struct_layouts_match_the_library():
    """The binding's ctypes structs have the library's sizes and field offsets."""
    L = fq.lib()
    fq._check_layout(L)
    assert int(L.flex_abi_layout(3, -1)) == ctypes.sizeof(fq.flex_kv_cache)
    assert int(L.flex_abi_layout(9, -1)) == -1


def test_layout_mismatch_is_refused(monkeypatch):
    """A binding struct that lacks a field the library has (here flex_kv_cache without
    valid_from) is refused before any call could pass it to the library."""
    class short_cache(ctypes.Structure):
        _fields_ = [f for f in fq.flex_kv_cache._fields_ if f[0] != "valid_from"]
    monkeypatch.setattr(fq, "_STRUCTS", (fq.flexq_config, fq.flexq_tensor, fq.flex_layer, short_cache))
    with pytest.raises(RuntimeError, match="layout"):
        fq._check_layout(fq.lib())
