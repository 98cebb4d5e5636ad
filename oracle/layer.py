"""OPT decoder layer, prefill (``mha``) and decode step (``mha_gen``) - oracle; test
infrastructure only.

Statement followed: the source-notes page «FlexGen» (PtirisNote), "Pytorch Backend" (``mha`` is the
prefill attention, ``mha_gen`` the decode attention) and "Flex Opt" (each
generation step runs load_cache, compute_layer, store_cache, so the key/value of
the current token are stored after the layer has run); the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南»,
section 6.3 (the KV cache is compressed with 4 bits, group 64, grouped along the
head dimension). The layer itself is the OPT pre-LayerNorm block:

    a   = LN(x; g1, b1)
    q   = (a Wq^T + bq) / sqrt(d),  k = a Wk^T + bk,  v = a Wv^T + bv
    o   = causal softmax attention of q over the keys/values, per head
    h1  = x + o Wo^T + bo
    out = h1 + ReLU(LN(h1; g2, b2) W1^T + b1) W2^T + b2

Readings (listed in the design notes): LayerNorm eps 1e-5 with biased variance;
fused QKV rows ordered [q; k; v] with feature = head * d + j; biases and LayerNorm
parameters fp16 and uncompressed; the 1/sqrt(d) factor applied after the query
bias; keys/values go through fp16 before they are quantised into the cache.

Arithmetic: float64 throughout, on the dequantised weights (the fp16 output of
``oracle.codec.decompress`` widened to float64). Only three roundings are part of
the definition: the weights' and the cache's fp16 dequantised values, the fp16
key/value handed to the cache quantiser, and the fp16 layer output. Matrix
products use numpy's matmul as a library primitive.
"""
from __future__ import annotations

import numpy as np

from . import codec

LN_EPS = 1e-5
W_CFG = dict(num_bits=4, group_size=64, group_dim=1)      # W[out][in], grouped along in


def layer_norm(x, g, b, eps=LN_EPS):
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * g + b, biased var."""
    x = np.asarray(x, dtype=np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps) * np.asarray(g, np.float64) + np.asarray(b, np.float64)


def softmax_rows(scores):
    """Max-subtracted softmax over the last axis; -inf entries get probability 0, and a
    row with no finite entry (nothing to attend to) gets all zeros."""
    s = np.asarray(scores, dtype=np.float64)
    m = s.max(axis=-1, keepdims=True)
    empty = ~np.isfinite(m)
    e = np.exp(s - np.where(empty, 0.0, m))
    z = e.sum(axis=-1, keepdims=True)
    return np.where(empty, 0.0, e / np.where(empty, 1.0, z))


def _key_visible(valid_from, batch, n_keys):
    """[b][1][1][n_keys] bool: key j of sequence b is a real token (j >= valid_from[b]).
    valid_from None: every key is."""
    if valid_from is None:
        return None
    vf = np.asarray(valid_from, np.int64).reshape(batch, 1, 1, 1)
    return np.arange(n_keys)[None, None, None, :] >= vf


ROW_BLOCK_ELEMS = 1 << 25      # weights are processed in blocks of whole rows of at most this many elements


def _row_blocks(rows, cols):
    """Row ranges [r0, r1) covering a [rows][cols] weight, each at most ROW_BLOCK_ELEMS elements.

    Groups run along the rows (group_dim 1), so blocks of whole rows are independent:
    blocking changes no result, it only bounds the host memory of the large layers."""
    step = max(1, ROW_BLOCK_ELEMS // max(1, cols))
    return [(r0, min(rows, r0 + step)) for r0 in range(0, rows, step)]


def compress_weights(raw, num_bits=4, group_size=64):
    """Quantise the four weight matrices of a raw parameter dict with the oracle codec.

    Returns a dict with the same keys; each weight is (codes, meta, shape)."""
    out = dict(raw)
    for k in ("w_qkv", "w_o", "w_fc1", "w_fc2"):
        w = np.asarray(raw[k])
        if w.dtype != np.float16:
            raise TypeError("weights must be float16")
        rows, cols = w.shape
        codes = np.empty((rows, cols * num_bits // 8), np.uint8)
        meta = np.empty((rows, cols // group_size, 2), np.float16)
        for r0, r1 in _row_blocks(rows, cols):
            codes[r0:r1], meta[r0:r1] = codec.compress(w[r0:r1], num_bits=num_bits, group_size=group_size,
                                                       group_dim=1)
        out[k] = (codes, meta, w.shape)
    return out


def dequant_weight(wq, num_bits=4, group_size=64, dtype=np.float64):
    """Dequantised weight [rows][cols]: the codec's fp16 output, widened to `dtype`
    (float16 keeps it as the codec returns it; every fp16 value is exact in float64)."""
    c, m, shape = wq
    rows, cols = shape
    out = np.empty(shape, dtype)
    for r0, r1 in _row_blocks(rows, cols):
        out[r0:r1] = codec.decompress(c[r0:r1], m[r0:r1], (r1 - r0, cols), num_bits=num_bits,
                                      group_size=group_size, group_dim=1)
    return out


def linear(a, w, bias=None):
    """a @ w.T (+ bias) in float64. w is a dense [out][in] weight (float64, or float16
    widened block by block, which gives the same products without a float64 copy of
    the whole matrix)."""
    a = np.asarray(a, np.float64)
    if w.dtype == np.float64:
        y = a @ w.T
    else:
        y = np.empty(a.shape[:-1] + (w.shape[0],), np.float64)
        for r0, r1 in _row_blocks(*w.shape):
            y[..., r0:r1] = a @ w[r0:r1].astype(np.float64).T
    if bias is not None:
        y += np.asarray(bias, np.float64)
    return y


class KVCache:
    """Compressed KV cache: codes [b][nh][max_seq][d*bits/8] uint8 and
    meta [b][nh][max_seq][d/gs][2] fp16 {min, scale}, for keys and for values.
    Quantised per (sequence, head, token) in groups along the head dimension."""

    def __init__(self, batch, n_heads, max_seq, head_dim, num_bits=4, group_size=64):
        self.b, self.nh, self.S, self.d = batch, n_heads, max_seq, head_dim
        self.bits, self.gs = num_bits, group_size
        cs = (batch, n_heads, max_seq, head_dim * num_bits // 8)
        ms = (batch, n_heads, max_seq, head_dim // group_size, 2)
        self.k_codes = np.zeros(cs, np.uint8)
        self.v_codes = np.zeros(cs, np.uint8)
        self.k_meta = np.zeros(ms, np.float16)
        self.v_meta = np.zeros(ms, np.float16)

    def _cfg(self):
        return dict(num_bits=self.bits, group_size=self.gs, group_dim=3)

    def store(self, k16, v16, pos0):
        """Quantise fp16 k/v [b][nh][n][d] into slots [pos0, pos0 + n)."""
        n = k16.shape[2]
        kc, km = codec.compress(np.asarray(k16, np.float16), **self._cfg())
        vc, vm = codec.compress(np.asarray(v16, np.float16), **self._cfg())
        self.k_codes[:, :, pos0:pos0 + n] = kc
        self.v_codes[:, :, pos0:pos0 + n] = vc
        self.k_meta[:, :, pos0:pos0 + n] = km
        self.v_meta[:, :, pos0:pos0 + n] = vm

    def load(self, n):
        """Dequantised fp16 keys and values of slots [0, n), as float64 [b][nh][n][d]."""
        shape = (self.b, self.nh, n, self.d)
        k = codec.decompress(self.k_codes[:, :, :n], self.k_meta[:, :, :n], shape, **self._cfg())
        v = codec.decompress(self.v_codes[:, :, :n], self.v_meta[:, :, :n], shape, **self._cfg())
        return k.astype(np.float64), v.astype(np.float64)


def _split_heads(t, n_heads):
    """[..., n, h] -> [..., nh, n, d] with feature = head * d + j."""
    *lead, n, h = t.shape
    d = h // n_heads
    t = t.reshape(*lead, n, n_heads, d)
    return np.moveaxis(t, -2, -3)


def _merge_heads(t):
    """[..., nh, n, d] -> [..., n, nh * d]."""
    t = np.moveaxis(t, -3, -2)
    *lead, n, nh, d = t.shape
    return t.reshape(*lead, n, nh * d)


def qkv_projection(x, P, Wqkv, n_heads):
    """LN1 and the fused QKV projection. x [b][n][h] -> q, k, v [b][nh][n][d] (q scaled)."""
    h = x.shape[-1]
    d = h // n_heads
    a = layer_norm(x, P["ln1_g"], P["ln1_b"])
    qkv = linear(a, Wqkv, P["b_qkv"])
    q = qkv[..., 0:h] / np.sqrt(d)
    k = qkv[..., h:2 * h]
    v = qkv[..., 2 * h:3 * h]
    return _split_heads(q, n_heads), _split_heads(k, n_heads), _split_heads(v, n_heads)


def attention_probs_prefill(q, k, valid_from=None):
    """Causal attention probabilities [b][nh][s][s]: row i over keys j <= i; with left
    padding (valid_from[b] = first real token of sequence b) only over keys
    valid_from[b] <= j <= i, and a pad row (i < valid_from[b]) attends to nothing."""
    s = q.shape[-2]
    scores = q @ np.swapaxes(k, -1, -2)
    mask = np.triu(np.ones((s, s), dtype=bool), k=1)
    vis = _key_visible(valid_from, q.shape[0], s)
    if vis is not None:
        mask = mask | ~vis
    scores = np.where(mask, -np.inf, scores)
    return softmax_rows(scores)


def mlp_block(x, o, P, W):
    """Output projection, residual, LN2, ReLU FFN, residual (all float64)."""
    h1 = np.asarray(x, np.float64) + linear(o, W["w_o"], P["b_o"])
    a2 = layer_norm(h1, P["ln2_g"], P["ln2_b"])
    f = np.maximum(linear(a2, W["w_fc1"], P["b_fc1"]), 0.0)
    out = h1 + linear(f, W["w_fc2"], P["b_fc2"])
    return out


def dequant_all(PQ, num_bits=4, group_size=64, dtype=np.float64):
    """The four dequantised weights; dtype=np.float16 keeps them at half the host memory
    of float32 (the large layers), with identical values."""
    return {k: dequant_weight(PQ[k], num_bits, group_size, dtype) for k in ("w_qkv", "w_o", "w_fc1", "w_fc2")}


def prefill_layer(x16, PQ, cache: KVCache, n_heads, W=None, valid_from=None):
    """Prefill (``mha``) over the prompt. x16 fp16 [b][s][h] -> fp16 [b][s][h].

    Attention reads the fresh float64 keys/values; the fp16 keys/values of every
    prompt token (pad tokens included) are quantised into cache slots [0, s).
    valid_from: optional [b] first real token of each left-padded prompt."""
    W = W if W is not None else dequant_all(PQ)
    x = np.asarray(x16, np.float64)
    q, k, v = qkv_projection(x, PQ, W["w_qkv"], n_heads)
    p = attention_probs_prefill(q, k, valid_from)
    o = _merge_heads(p @ v)
    out = mlp_block(x, o, PQ, W)
    cache.store(k.astype(np.float16), v.astype(np.float16), 0)
    return out.astype(np.float16)


def decode_layer(x16, PQ, cache: KVCache, pos, n_heads, W=None, valid_from=None):
    """Decode step (``mha_gen``) at position pos. x16 fp16 [b][h] -> fp16 [b][h].

    The new token attends to the dequantised cache slots [0, pos) and to its own
    fresh float64 key/value at pos; afterwards its fp16 key/value are quantised into
    slot pos. With left padding (valid_from[b]) the slots below valid_from[b] are not
    attended. Sequences are independent, so a cache holding a subset of a batch gives
    that subset's rows of the full result."""
    W = W if W is not None else dequant_all(PQ)
    x = np.asarray(x16, np.float64)[:, None, :]             # [b][1][h]
    q, k, v = qkv_projection(x, PQ, W["w_qkv"], n_heads)    # [b][nh][1][d]
    kc, vc = cache.load(pos)                                # [b][nh][pos][d]
    keys = np.concatenate([kc, k], axis=2)
    vals = np.concatenate([vc, v], axis=2)
    scores = q @ np.swapaxes(keys, -1, -2)                  # [b][nh][1][pos+1]
    vis = _key_visible(valid_from, x.shape[0], pos + 1)
    if vis is not None:
        vis = vis | (np.arange(pos + 1) == pos)             # the new token itself is real
        scores = np.where(vis, scores, -np.inf)
    p = softmax_rows(scores)
    o = _merge_heads(p @ vals)                              # [b][1][h]
    out = mlp_block(x, o, PQ, W)[:, 0, :]
    cache.store(k.astype(np.float16), v.astype(np.float16), pos)
    return out.astype(np.float16)


def decode_attention(q16, k_new16, v_new16, cache: KVCache, pos, valid_from=None):
    """Decode attention alone: q, k_new, v_new fp16 [b][nh][d] (q already scaled).

    Returns o float64 [b][nh][d] = softmax(q . [cache[vf,pos); k_new]) [cache[vf,pos); v_new]
    with vf = valid_from[b] (0 without padding)."""
    q = np.asarray(q16, np.float64)[:, :, None, :]
    kn = np.asarray(k_new16, np.float64)[:, :, None, :]
    vn = np.asarray(v_new16, np.float64)[:, :, None, :]
    kc, vc = cache.load(pos)
    keys = np.concatenate([kc, kn], axis=2)
    vals = np.concatenate([vc, vn], axis=2)
    scores = q @ np.swapaxes(keys, -1, -2)
    vis = _key_visible(valid_from, q.shape[0], pos + 1)
    if vis is not None:
        scores = np.where(vis | (np.arange(pos + 1) == pos), scores, -np.inf)
    p = softmax_rows(scores)
    return (p @ vals)[:, :, 0, :]


def prefill_attention(q16, k16, v16, valid_from=None):
    """Prefill attention alone on fp16 q/k/v [b][s][nh][d] (q already scaled) -> float64 o."""
    q = np.moveaxis(np.asarray(q16, np.float64), 2, 1)
    k = np.moveaxis(np.asarray(k16, np.float64), 2, 1)
    v = np.moveaxis(np.asarray(v16, np.float64), 2, 1)
    o = attention_probs_prefill(q, k, valid_from) @ v
    return np.moveaxis(o, 1, 2)
