"""Python binding of the flexq C ABI (``include/flexq.h``).

Argument marshalling only: every step of the hot path runs in the CUDA kernels of
``libflexq.so``. PyTorch provides device memory and streams. There is no fallback:
if the library is missing, every call raises.

The names mirror the C entry points. Tensors are torch CUDA tensors; outputs that
are not given are allocated with torch.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflexq.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "flexq.h")

FLEX_OK = 0
FLEX_ERR_INVALID_ARG = -1
FLEX_ERR_UNSUPPORTED = -2
FLEX_ERR_SHAPE = -3
FLEX_ERR_ALIGN = -4
FLEX_ERR_WORKSPACE = -5
FLEX_ERR_CUDA = -6
FLEX_ERR_TIMEOUT = -7
FLEX_ERR_SCRATCH_LIMIT = -8

FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES = 8 << 20

FLEX_GEMM_X_INTERLEAVED = 0x10

FLEX_EPI_NONE = 0
FLEX_EPI_RELU = 1
FLEX_EPI_RESIDUAL = 2


class FlexError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


# ---- C structs -------------------------------------------------------------------
class flexq_config(ctypes.Structure):
    _fields_ = [("num_bits", ctypes.c_int32), ("group_size", ctypes.c_int32),
                ("group_dim", ctypes.c_int32), ("symmetric", ctypes.c_int32)]


class flexq_tensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("cfg", flexq_config)]


class flex_layer(ctypes.Structure):
    _fields_ = [("h", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ffn", ctypes.c_int32),
                ("ln1_g", ctypes.c_void_p), ("ln1_b", ctypes.c_void_p),
                ("ln2_g", ctypes.c_void_p), ("ln2_b", ctypes.c_void_p),
                ("w_qkv", flexq_tensor), ("w_o", flexq_tensor), ("w_fc1", flexq_tensor),
                ("w_fc2", flexq_tensor),
                ("b_qkv", ctypes.c_void_p), ("b_o", ctypes.c_void_p), ("b_fc1", ctypes.c_void_p),
                ("b_fc2", ctypes.c_void_p)]


class flex_kv_cache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_meta", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_meta", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("max_seq", ctypes.c_int32), ("cfg", flexq_config), ("valid_from", ctypes.c_void_p)]


_I32, _I64, _P = ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
_SIGS = {
    "flexq_codes_bytes": (_I64, [_I32, ctypes.POINTER(ctypes.c_int64), flexq_config]),
    "flexq_meta_bytes": (_I64, [_I32, ctypes.POINTER(ctypes.c_int64), flexq_config]),
    "flexq_compress": (_I32, [_P, _I32, ctypes.POINTER(ctypes.c_int64), flexq_config, _P, _P, _P]),
    "flexq_decompress": (_I32, [_P, _P, _I32, ctypes.POINTER(ctypes.c_int64), flexq_config, _P, _P]),
    "flex_workspace_bytes": (_I64, [ctypes.POINTER(flex_layer), _I32, _I32]),
    "flex_prefill_layer": (_I32, [ctypes.POINTER(flex_layer), ctypes.POINTER(flex_kv_cache), _P, _P,
                                  _I32, _I32, _P, _I64, _P]),
    "flex_decode_layer": (_I32, [ctypes.POINTER(flex_layer), ctypes.POINTER(flex_kv_cache), _P, _P,
                                 _I32, _I32, _P, _I64, _P]),
    "flex_prefill_layer_batches": (_I32, [ctypes.POINTER(flex_layer), ctypes.POINTER(flex_kv_cache), _I32, _P, _P,
                                          _I32, _I32, _P, _I64, _P]),
    "flex_decode_layer_batches": (_I32, [ctypes.POINTER(flex_layer), ctypes.POINTER(flex_kv_cache), _I32, _P, _P,
                                         _I32, _I32, _P, _I64, _P]),
    "flex_append_kv": (_I32, [ctypes.POINTER(flex_kv_cache), _P, _P, _I64, _I32, _I32, _P]),
    "flex_decode_attention_ws_bytes": (_I64, [ctypes.POINTER(flex_kv_cache), _I32, _I32]),
    "flex_decode_attention": (_I32, [ctypes.POINTER(flex_kv_cache), _P, _P, _P, _I64, _P, _I32, _I32,
                                     _P, _I64, _P]),
    "flex_decode_attention_noalloc": (_I32, [ctypes.POINTER(flex_kv_cache), _P, _P, _P, _I64, _P, _I32,
                                             _I32, _P]),
    "flex_prefill_attention": (_I32, [_P, _P, _P, _I64, _P, _I32, _I32, _I32, _I32, _P, _P]),
    "flex_gemm_ws_bytes": (_I64, [_I32, _I32, _I32]),
    "flex_dequant_gemm": (_I32, [_P, ctypes.POINTER(flexq_tensor), _P, _P, _P, _I32, _I32, _P, _I64, _P]),
    "flex_layernorm": (_I32, [_P, _P, _P, _P, _I64, _I32, _P]),
    "flex_embed": (_I32, [ctypes.POINTER(flexq_tensor), _I32, _P, _I32, _P, _P, _I64, _P, _P]),
    "flex_lm_head_ws_bytes": (_I64, [ctypes.POINTER(flexq_tensor), _I32, _I64, _I32]),
    "flex_lm_head_argmax": (_I32, [ctypes.POINTER(flexq_tensor), _I32, _P, _P, _P, _I64, _P, _P, _P, _I64, _P]),
    "flex_get_status": (_I32, [_P]),
    "flex_set_wait_limit_ns": (ctypes.c_uint64, [ctypes.c_uint64]),
    "flex_set_gemm_gate": (_P, [_P]),
    "flex_gemm_plan": (_I32, [_I32, _I32, _I32, _I32, _P]),
    "flex_set_gemm_streamk": (_I32, [_I32]),
    "flex_set_gemm_gemv": (_I32, [_I32]),
    "flex_status_string": (ctypes.c_char_p, [_I32]),
    "flex_abi_layout": (_I64, [_I32, _I32]),
}

_STRUCTS = (flexq_config, flexq_tensor, flex_layer, flex_kv_cache)   # flex_abi_layout's `which` order


def _check_layout(L):
    """Refuse a library whose struct layouts differ from the ctypes declarations here: a
    mismatch would make the library read past (or misread) the structs this module
    passes, and hand the kernels wrong pointers."""
    for which, S in enumerate(_STRUCTS):
        fields = [f[0] for f in S._fields_]
        theirs = [int(L.flex_abi_layout(which, -1))] + [int(L.flex_abi_layout(which, i)) for i in range(len(fields))]
        ours = [ctypes.sizeof(S)] + [getattr(S, f).offset for f in fields]
        extra = int(L.flex_abi_layout(which, len(fields)))
        if theirs != ours or extra != -1:
            raise RuntimeError(f"libflexq.so struct layout of {S.__name__} differs from the binding "
                               f"(library {theirs}, binding {ours}); rebuild the library")

_lib = None


def lib():
    """The loaded libflexq.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libflexq.so is missing ({LIB_PATH}); build it with "
                               "`python -m group_wise_int4_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name, None)
            if fn is None:
                continue
            fn.restype = res
            fn.argtypes = args
        _check_layout(L)
        _lib = L
    return _lib


def declared_functions(header: str = HEADER_PATH):
    """Names of the functions declared in include/flexq.h."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(flexq?_\w+)\s*\(", text)))


def status_string(code: int) -> str:
    try:
        return lib().flex_status_string(int(code)).decode()
    except Exception:
        return "status"


def _check(code: int, what: str):
    if code != FLEX_OK:
        raise FlexError(code, what)


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream or 0)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape_arr(shape):
    arr = (ctypes.c_int64 * 4)()
    for i, d in enumerate(shape):
        arr[i] = int(d)
    return arr


def config(num_bits=4, group_size=64, group_dim=0, symmetric=0) -> flexq_config:
    return flexq_config(int(num_bits), int(group_size), int(group_dim), int(symmetric))


# ---- codec -----------------------------------------------------------------------
def codes_shape(shape, cfg: flexq_config):
    """Packed codes: num_groups * group_size * bits / 8 bytes along group_dim."""
    shape = tuple(int(d) for d in shape)
    gd = cfg.group_dim % len(shape)
    ng = -(-shape[gd] // cfg.group_size)
    return shape[:gd] + (ng * cfg.group_size * cfg.num_bits // 8,) + shape[gd + 1:]


def meta_shape(shape, cfg: flexq_config):
    """Metadata shape in fp16 units: one {min, scale} pair per group as a trailing 2."""
    shape = tuple(int(d) for d in shape)
    gd = cfg.group_dim % len(shape)
    return shape[:gd] + (-(-shape[gd] // cfg.group_size),) + shape[gd + 1:] + (2,)


def flexq_codes_bytes(shape, cfg: flexq_config) -> int:
    return int(lib().flexq_codes_bytes(len(shape), _shape_arr(shape), cfg))


def flexq_meta_bytes(shape, cfg: flexq_config) -> int:
    return int(lib().flexq_meta_bytes(len(shape), _shape_arr(shape), cfg))


def flexq_compress(x: torch.Tensor, cfg: flexq_config, codes=None, meta=None, stream=None):
    """Compress fp16 CUDA tensor x; returns (codes uint8, meta fp16 [..., 2])."""
    shape = tuple(x.shape)
    if codes is None:
        codes = torch.empty(codes_shape(shape, cfg), dtype=torch.uint8, device=x.device)
    if meta is None:
        meta = torch.empty(meta_shape(shape, cfg), dtype=torch.float16, device=x.device)
    rc = lib().flexq_compress(_ptr(x), len(shape), _shape_arr(shape), cfg, _ptr(codes), _ptr(meta),
                              ctypes.c_void_p(_stream(stream)))
    _check(rc, "flexq_compress")
    return codes, meta


def flexq_decompress(codes: torch.Tensor, meta: torch.Tensor, shape, cfg: flexq_config, y=None,
                     stream=None):
    shape = tuple(int(d) for d in shape)
    if y is None:
        y = torch.empty(shape, dtype=torch.float16, device=codes.device)
    rc = lib().flexq_decompress(_ptr(codes), _ptr(meta), len(shape), _shape_arr(shape), cfg, _ptr(y),
                                ctypes.c_void_p(_stream(stream)))
    _check(rc, "flexq_decompress")
    return y


# ---- compressed weights, layer parameters, KV cache ---------------------------------
class CompressedWeight:
    """A weight W[out][in] compressed along `in` (group_dim 1) on the device."""

    def __init__(self, w: torch.Tensor, num_bits=4, group_size=64, stream=None):
        assert w.dim() == 2 and w.dtype == torch.float16 and w.is_cuda
        self.shape = tuple(w.shape)
        self.cfg = config(num_bits, group_size, 1)
        self.codes, self.meta = flexq_compress(w.contiguous(), self.cfg, stream=stream)

    def struct(self) -> flexq_tensor:
        t = flexq_tensor()
        t.codes = self.codes.data_ptr()
        t.meta = self.meta.data_ptr()
        t.ndim = 2
        t.shape[0], t.shape[1] = self.shape
        t.cfg = self.cfg
        return t

    def nbytes(self) -> int:
        return self.codes.numel() + self.meta.numel() * 2


class FlexLayer:
    """Device parameters of one OPT decoder layer (weights compressed on the GPU with
    flexq_compress, biases and LayerNorm parameters fp16)."""

    def __init__(self, raw: dict, n_heads: int, num_bits=4, group_size=64, device="cuda", stream=None):
        dev = lambda t: t.to(device=device, dtype=torch.float16).contiguous()
        self.h = int(raw["w_o"].shape[0])
        self.ffn = int(raw["w_fc1"].shape[0])
        self.n_heads = int(n_heads)
        self.head_dim = self.h // self.n_heads
        self.vec = {k: dev(raw[k]) for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_qkv", "b_o",
                                             "b_fc1", "b_fc2")}
        self.w = {k: CompressedWeight(dev(raw[k]), num_bits, group_size, stream=stream)
                  for k in ("w_qkv", "w_o", "w_fc1", "w_fc2")}
        self._struct = None

    def struct(self) -> flex_layer:
        if self._struct is None:
            s = flex_layer()
            s.h, s.n_heads, s.head_dim, s.ffn = self.h, self.n_heads, self.head_dim, self.ffn
            for k, v in self.vec.items():
                setattr(s, k, v.data_ptr())
            for k, w in self.w.items():
                setattr(s, k, w.struct())
            self._struct = s
        return self._struct

    def weight_bytes(self) -> int:
        return sum(w.nbytes() for w in self.w.values())


class FlexKVCache:
    """Compressed KV cache of one layer: codes [b][nh][max_seq][d*bits/8] uint8 and
    meta [b][nh][max_seq][d/gs][2] fp16 for keys and values. valid_from: optional int32
    CUDA tensor [b] of left-padding starts (first real token of each sequence)."""

    def __init__(self, batch, n_heads, head_dim, max_seq, num_bits=4, group_size=64, device="cuda",
                 valid_from: Optional[torch.Tensor] = None):
        self.batch, self.n_heads, self.head_dim, self.max_seq = batch, n_heads, head_dim, max_seq
        self.valid_from = valid_from
        self.cfg = config(num_bits, group_size, 3)
        cs = (batch, n_heads, max_seq, head_dim * num_bits // 8)
        ms = (batch, n_heads, max_seq, head_dim // group_size, 2)
        self.k_codes = torch.zeros(cs, dtype=torch.uint8, device=device)
        self.v_codes = torch.zeros(cs, dtype=torch.uint8, device=device)
        self.k_meta = torch.zeros(ms, dtype=torch.float16, device=device)
        self.v_meta = torch.zeros(ms, dtype=torch.float16, device=device)
        self._struct = None

    def struct(self) -> flex_kv_cache:
        if self._struct is None:
            s = flex_kv_cache()
            s.k_codes, s.k_meta = self.k_codes.data_ptr(), self.k_meta.data_ptr()
            s.v_codes, s.v_meta = self.v_codes.data_ptr(), self.v_meta.data_ptr()
            s.batch, s.n_heads, s.head_dim, s.max_seq = self.batch, self.n_heads, self.head_dim, self.max_seq
            s.cfg = self.cfg
            self._struct = s
        self._struct.valid_from = None if self.valid_from is None else self.valid_from.data_ptr()
        return self._struct

    def fill_from(self, k16: torch.Tensor, v16: torch.Tensor, stream=None):
        """Quantise fp16 histories [b][nh][n][d] into slots [0, n) with flexq_compress."""
        n = k16.shape[2]
        for src, codes, meta in ((k16, self.k_codes, self.k_meta), (v16, self.v_codes, self.v_meta)):
            c, m = flexq_compress(src.contiguous(), self.cfg, stream=stream)
            codes[:, :, :n].copy_(c)
            meta[:, :, :n].copy_(m)


# ---- layer calls -------------------------------------------------------------------
def flex_workspace_bytes(layer: FlexLayer, batch: int, seq: int) -> int:
    return int(lib().flex_workspace_bytes(ctypes.byref(layer.struct()), int(batch), int(seq)))


def flex_prefill_layer(layer: FlexLayer, cache: FlexKVCache, x_in, x_out, batch, seq, ws, stream=None):
    rc = lib().flex_prefill_layer(ctypes.byref(layer.struct()), ctypes.byref(cache.struct()), _ptr(x_in),
                                  _ptr(x_out), int(batch), int(seq), _ptr(ws),
                                  int(ws.numel() * ws.element_size()), ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_prefill_layer")


def flex_decode_layer(layer: FlexLayer, cache: FlexKVCache, x_in, x_out, batch, pos, ws, stream=None):
    rc = lib().flex_decode_layer(ctypes.byref(layer.struct()), ctypes.byref(cache.struct()), _ptr(x_in),
                                 _ptr(x_out), int(batch), int(pos), _ptr(ws),
                                 int(ws.numel() * ws.element_size()), ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_decode_layer")


def _cache_array(caches):
    arr = (flex_kv_cache * len(caches))()
    for i, c in enumerate(caches):
        arr[i] = c.struct()
    return arr


def flex_prefill_layer_batches(layer: FlexLayer, caches, x_in, x_out, batch, seq, ws, stream=None):
    """len(caches) gpu-batches of `batch` sequences through one layer, one weight pass."""
    arr = _cache_array(caches)
    rc = lib().flex_prefill_layer_batches(ctypes.byref(layer.struct()), arr, len(caches), _ptr(x_in), _ptr(x_out),
                                          int(batch), int(seq), _ptr(ws), int(ws.numel() * ws.element_size()),
                                          ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_prefill_layer_batches")


def flex_decode_layer_batches(layer: FlexLayer, caches, x_in, x_out, batch, pos, ws, stream=None):
    """Decode step of len(caches) gpu-batches of `batch` sequences, one weight pass."""
    arr = _cache_array(caches)
    rc = lib().flex_decode_layer_batches(ctypes.byref(layer.struct()), arr, len(caches), _ptr(x_in), _ptr(x_out),
                                         int(batch), int(pos), _ptr(ws), int(ws.numel() * ws.element_size()),
                                         ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_decode_layer_batches")


def flex_append_kv(cache: FlexKVCache, k_new, v_new, row_stride, batch, pos, stream=None):
    rc = lib().flex_append_kv(ctypes.byref(cache.struct()), _ptr(k_new), _ptr(v_new), int(row_stride),
                              int(batch), int(pos), ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_append_kv")


def flex_decode_attention_ws_bytes(cache: FlexKVCache, batch, pos) -> int:
    return int(lib().flex_decode_attention_ws_bytes(ctypes.byref(cache.struct()), int(batch), int(pos)))


def flex_decode_attention(cache: FlexKVCache, q, k_new, v_new, row_stride, o, batch, pos, ws,
                          stream=None):
    rc = lib().flex_decode_attention(ctypes.byref(cache.struct()), _ptr(q), _ptr(k_new), _ptr(v_new),
                                     int(row_stride), _ptr(o), int(batch), int(pos), _ptr(ws),
                                     int(ws.numel() * ws.element_size()) if ws is not None else 0,
                                     ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_decode_attention")


def flex_decode_attention_noalloc(cache: FlexKVCache, q, k_new, v_new, row_stride, o, batch, pos,
                                  stream=None):
    """flex_decode_attention with the library's built-in scratch instead of a workspace
    (no device allocation; calls that may overlap on one device race on that scratch)."""
    rc = lib().flex_decode_attention_noalloc(ctypes.byref(cache.struct()), _ptr(q), _ptr(k_new), _ptr(v_new),
                                             int(row_stride), _ptr(o), int(batch), int(pos),
                                             ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_decode_attention_noalloc")


def flex_prefill_attention(q, k, v, row_stride, o, batch, seq, n_heads, head_dim, valid_from=None, stream=None):
    rc = lib().flex_prefill_attention(_ptr(q), _ptr(k), _ptr(v), int(row_stride), _ptr(o), int(batch),
                                      int(seq), int(n_heads), int(head_dim), _ptr(valid_from),
                                      ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_prefill_attention")


def flex_gemm_ws_bytes(M, N, K) -> int:
    return int(lib().flex_gemm_ws_bytes(int(M), int(N), int(K)))


def flex_dequant_gemm(x, W: CompressedWeight, bias, residual, y, M, epilogue, ws, stream=None):
    st = W.struct()
    rc = lib().flex_dequant_gemm(_ptr(x), ctypes.byref(st), _ptr(bias), _ptr(residual), _ptr(y), int(M),
                                 int(epilogue), _ptr(ws),
                                 int(ws.numel() * ws.element_size()) if ws is not None else 0,
                                 ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_dequant_gemm")


def flex_layernorm(x, g, b, y, rows, h, stream=None):
    rc = lib().flex_layernorm(_ptr(x), _ptr(g), _ptr(b), _ptr(y), int(rows), int(h),
                              ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_layernorm")


# ---- whole model: embedding, output head, greedy choice ------------------------------
def flex_embed(E: "CompressedWeight", vocab, P, tokens, positions, x=None, stream=None):
    """x [n][h] fp16 = E^[tokens] + P[positions] (tokens/positions: int32 CUDA tensors)."""
    n = int(tokens.numel())
    if x is None:
        x = torch.empty((n, E.shape[1]), dtype=torch.float16, device=tokens.device)
    rc = lib().flex_embed(ctypes.byref(E.struct()), int(vocab), _ptr(P), int(P.shape[0]), _ptr(tokens),
                          _ptr(positions), n, _ptr(x), ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_embed")
    return x


def flex_lm_head_ws_bytes(E: "CompressedWeight", vocab, n, with_logits=False) -> int:
    return int(lib().flex_lm_head_ws_bytes(ctypes.byref(E.struct()), int(vocab), int(n), int(bool(with_logits))))


def flex_lm_head_argmax(E: "CompressedWeight", vocab, lnf_g, lnf_b, x, ws, next_ids=None, logits=None,
                        stream=None):
    """Greedy next tokens (int32 [n]) of the rows of x; logits (fp16 [n][V_pad]) if given."""
    n = int(x.shape[0])
    if next_ids is None:
        next_ids = torch.empty(n, dtype=torch.int32, device=x.device)
    rc = lib().flex_lm_head_argmax(ctypes.byref(E.struct()), int(vocab), _ptr(lnf_g), _ptr(lnf_b), _ptr(x), n,
                                   _ptr(next_ids), _ptr(logits), _ptr(ws), int(ws.numel() * ws.element_size()),
                                   ctypes.c_void_p(_stream(stream)))
    _check(rc, "flex_lm_head_argmax")
    return next_ids


def flex_abi_layout(which: int, field: int) -> int:
    return int(lib().flex_abi_layout(int(which), int(field)))


def flex_set_wait_limit_ns(ns: int) -> int:
    """Limit of the GEMM's pipeline waits for later launches (0 = default 2 s); returns the old one."""
    return int(lib().flex_set_wait_limit_ns(int(ns)))


def flex_gemm_plan(M: int, N: int, K: int, bits: int = 4) -> dict:
    """The launch plan of flex_dequant_gemm for this problem on the current device."""
    out = (ctypes.c_int32 * 4)()
    _check(lib().flex_gemm_plan(int(M), int(N), int(K), int(bits), ctypes.cast(out, ctypes.c_void_p)), "flex_gemm_plan")
    return {"kernel": ("gemv", "tc128", "tc256")[out[0]], "tiles": out[1], "splits": out[2],
            "reduce": "none" if out[2] == 1 and out[3] == 0 else ("ticket", "cluster", "streamk", "exchange")[out[3]]}


def flex_set_gemm_streamk(enable: bool) -> bool:
    """Stream-K schedule of the 256-row GEMM for later plans; returns the previous setting."""
    return bool(lib().flex_set_gemm_streamk(1 if enable else 0))


def flex_set_gemm_gemv(enable: bool) -> bool:
    """Small-batch GEMV route for later launches; returns the previous setting."""
    return bool(lib().flex_set_gemm_gemv(1 if enable else 0))


def flex_set_gemm_gate(gate) -> int:
    """Gate of the tensor-core GEMM's weight loads for later launches (a device int32
    tensor, or None to remove it); returns the previous gate's address (0 if none)."""
    prev = lib().flex_set_gemm_gate(None if gate is None else _ptr(gate))
    return int(prev or 0)


def flex_get_status(stream=None) -> int:
    return int(lib().flex_get_status(ctypes.c_void_p(_stream(stream))))


def flex_status_string(code: int) -> str:
    return lib().flex_status_string(int(code)).decode()
