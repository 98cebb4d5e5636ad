"""Python access to the plain C++17 fp32 oracle (``oracle/cpp/flexq_oracle.cpp``); test
infrastructure only.

The C++ oracle is a second statement of the method, independent of both the CUDA
library and the numpy oracle: the group-wise min/max quantiser of the walkthrough page
«FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3, and the OPT layer (``mha`` prefill and ``mha_gen``
decode step of the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend" / "Flex
Opt") in IEEE binary32. It is compiled on first use with g++ (-O2 -ffp-contract=off, so
no multiply-add is fused) into ``oracle/libflexq_oracle.so``. This module only moves
numpy arrays in and out.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_DIR = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_DIR, "cpp", "flexq_oracle.cpp")
LIB_PATH = os.path.join(_DIR, "libflexq_oracle.so")
CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fPIC", "-shared", "-pthread"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the C++ oracle (when the library is missing or older than its source)."""
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(SRC):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        r = subprocess.run(["g++"] + CXXFLAGS + [SRC, "-o", tmp], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"g++ failed for the C++ oracle:\n{r.stdout}\n{r.stderr}")
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


class _Desc(ctypes.Structure):
    _fields_ = [("h", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int), ("ffn", ctypes.c_int),
                ("w_bits", ctypes.c_int)] + \
               [(k, ctypes.c_void_p) for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_qkv", "b_o", "b_fc1", "b_fc2")] + \
               [("w_codes", ctypes.c_void_p * 4), ("w_meta", ctypes.c_void_p * 4)]


class _Cache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("v_codes", ctypes.c_void_p), ("k_meta", ctypes.c_void_p),
                ("v_meta", ctypes.c_void_p), ("batch", ctypes.c_int), ("n_heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("max_seq", ctypes.c_int), ("bits", ctypes.c_int), ("gs", ctypes.c_int)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, I64P = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(ctypes.c_int64)
        L.fo_half_to_float.restype, L.fo_half_to_float.argtypes = ctypes.c_float, [ctypes.c_uint16]
        L.fo_float_to_half.restype, L.fo_float_to_half.argtypes = ctypes.c_uint16, [ctypes.c_float]
        L.fo_float_to_half_n.restype = None
        L.fo_float_to_half_n.argtypes = [P, ctypes.c_int64, P]
        L.fo_compress.restype, L.fo_compress.argtypes = I, [P, I, I64P, I, I, I, P, P, I]
        L.fo_decompress.restype, L.fo_decompress.argtypes = I, [P, P, I, I64P, I, I, I, P, I]
        L.fo_layer_new.restype, L.fo_layer_new.argtypes = P, [ctypes.POINTER(_Desc), I]
        L.fo_layer_free.restype, L.fo_layer_free.argtypes = None, [P]
        for fn in (L.fo_prefill_layer, L.fo_decode_layer):
            fn.restype, fn.argtypes = I, [P, ctypes.POINTER(_Cache), P, I, I, P, I]
        L.fo_decode_attention.restype = I
        L.fo_decode_attention.argtypes = [ctypes.POINTER(_Cache), P, P, P, I, I, P]
        _lib = L
    return _lib


def threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0)) or 1
    except AttributeError:
        return os.cpu_count() or 1


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


def _shape(shape):
    return (ctypes.c_int64 * len(shape))(*[int(d) for d in shape])


def half_to_float(bits: int) -> float:
    return float(lib().fo_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(lib().fo_float_to_half(float(x)))


def float_to_half_array(x) -> np.ndarray:
    """float32 array -> its fp16 bit patterns (uint16), rounded by the oracle's converter."""
    f = np.ascontiguousarray(x, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().fo_float_to_half_n(_p(f), f.size, _p(out))
    return out


def codes_shape(shape, num_bits, group_size, group_dim):
    gd = group_dim % len(shape)
    return tuple(shape[:gd]) + (shape[gd] * num_bits // 8,) + tuple(shape[gd + 1:])


def meta_shape(shape, group_size, group_dim):
    gd = group_dim % len(shape)
    return tuple(shape[:gd]) + (shape[gd] // group_size,) + tuple(shape[gd + 1:]) + (2,)


def compress(x16, num_bits=4, group_size=64, group_dim=0, nthreads=None):
    """Compress a float16 array; returns (codes uint8, meta float16 [..., 2] = {min, scale})."""
    x = np.ascontiguousarray(x16)
    if x.dtype != np.float16:
        raise TypeError("input must be float16")
    codes = np.empty(codes_shape(x.shape, num_bits, group_size, group_dim), np.uint8)
    meta = np.empty(meta_shape(x.shape, group_size, group_dim), np.float16)
    rc = lib().fo_compress(_p(x), x.ndim, _shape(x.shape), num_bits, group_size, group_dim, _p(codes), _p(meta),
                           nthreads or threads())
    if rc != 0:
        raise ValueError("unsupported configuration or shape")
    return codes, meta


def decompress(codes, meta, shape, num_bits=4, group_size=64, group_dim=0, nthreads=None):
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    m = np.ascontiguousarray(meta, dtype=np.float16)
    y = np.empty(tuple(int(d) for d in shape), np.float16)
    rc = lib().fo_decompress(_p(c), _p(m), y.ndim, _shape(y.shape), num_bits, group_size, group_dim, _p(y),
                             nthreads or threads())
    if rc != 0:
        raise ValueError("unsupported configuration or shape")
    return y


class KVCache:
    """Compressed KV cache in the library's layout: codes [b][nh][max_seq][d*bits/8],
    meta [b][nh][max_seq][d/gs][2] fp16, for keys and for values."""

    def __init__(self, batch, n_heads, max_seq, head_dim, num_bits=4, group_size=64):
        self.b, self.nh, self.S, self.d, self.bits, self.gs = batch, n_heads, max_seq, head_dim, num_bits, group_size
        cs = (batch, n_heads, max_seq, head_dim * num_bits // 8)
        ms = (batch, n_heads, max_seq, head_dim // group_size, 2)
        self.k_codes = np.zeros(cs, np.uint8)
        self.v_codes = np.zeros(cs, np.uint8)
        self.k_meta = np.zeros(ms, np.float16)
        self.v_meta = np.zeros(ms, np.float16)

    def struct(self):
        return _Cache(self.k_codes.ctypes.data, self.v_codes.ctypes.data, self.k_meta.ctypes.data,
                      self.v_meta.ctypes.data, self.b, self.nh, self.d, self.S, self.bits, self.gs)


class Layer:
    """One OPT layer in the C++ oracle: the four weights compressed with the C++ codec
    (group 64 along the input dimension) and dequantised once inside the library."""

    def __init__(self, raw, n_heads, num_bits=4, nthreads=None):
        h = int(raw["w_o"].shape[0])
        ffn = int(raw["w_fc1"].shape[0])
        self.h, self.nh, self.d, self.ffn = h, int(n_heads), h // int(n_heads), ffn
        self._keep = []
        d = _Desc()
        d.h, d.n_heads, d.head_dim, d.ffn, d.w_bits = h, self.nh, self.d, ffn, num_bits
        for k in ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_qkv", "b_o", "b_fc1", "b_fc2"):
            a = np.ascontiguousarray(np.asarray(raw[k], np.float16))
            self._keep.append(a)
            setattr(d, k, a.ctypes.data)
        for i, k in enumerate(("w_qkv", "w_o", "w_fc1", "w_fc2")):
            c, m = compress(np.asarray(raw[k], np.float16), num_bits, 64, 1, nthreads)
            self._keep += [c, m]
            d.w_codes[i] = c.ctypes.data
            d.w_meta[i] = m.ctypes.data
        self._h = lib().fo_layer_new(ctypes.byref(d), nthreads or threads())
        if not self._h:
            raise ValueError("bad layer description")
        self._keep = []                         # the library holds its own dequantised copy

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            try:
                _lib.fo_layer_free(h)
            except Exception:          # interpreter shutdown
                pass


def prefill_layer(x16, layer: Layer, cache: KVCache, nthreads=None):
    """x16 float16 [b][s][h] -> float16 [b][s][h]; writes cache slots [0, s)."""
    x = np.ascontiguousarray(x16, np.float16)
    b, s, _ = x.shape
    out = np.empty_like(x)
    st = cache.struct()
    rc = lib().fo_prefill_layer(layer._h, ctypes.byref(st), _p(x), b, s, _p(out), nthreads or threads())
    if rc != 0:
        raise ValueError("bad prefill arguments")
    return out


def decode_layer(x16, layer: Layer, cache: KVCache, pos, nthreads=None):
    """x16 float16 [b][h] -> float16 [b][h] at position pos (writes cache slot pos)."""
    x = np.ascontiguousarray(x16, np.float16)
    b = x.shape[0]
    out = np.empty_like(x)
    st = cache.struct()
    rc = lib().fo_decode_layer(layer._h, ctypes.byref(st), _p(x), b, int(pos), _p(out), nthreads or threads())
    if rc != 0:
        raise ValueError("bad decode arguments")
    return out


def decode_attention(q16, k16, v16, cache: KVCache, pos):
    """q, k_new, v_new float16 [b][nh][d] -> o float32 [b][nh][d]."""
    q = np.ascontiguousarray(q16, np.float16)
    k = np.ascontiguousarray(k16, np.float16)
    v = np.ascontiguousarray(v16, np.float16)
    o = np.empty(q.shape, np.float32)
    st = cache.struct()
    rc = lib().fo_decode_attention(ctypes.byref(st), _p(q), _p(k), _p(v), q.shape[0], int(pos), _p(o))
    if rc != 0:
        raise ValueError("bad decode attention arguments")
    return o
