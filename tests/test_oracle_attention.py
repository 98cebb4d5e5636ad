"""Pins of the oracle's stand-alone attention functions, which the GPU attention parity
tests compare against: ``oracle.layer.decode_attention`` (``mha_gen``: the new token
over the dequantised cache slots [0, pos) plus its own fresh key/value) and
``oracle.layer.prefill_attention`` (``mha``: causal attention on fresh q/k/v laid out
[batch][seq][heads][head_dim]).

Each pin is something other than the oracle restated: a one-entry softmax, uniform
attention over exactly representable keys (the plain mean of the values), causality,
and pure-Python loops that decompress every cache slot on their own (so a wrong slot
count, a dropped fresh key or a transposed layout fails).
"""
import math

import numpy as np
import pytest

import synth
from oracle import codec, layer


def _rand16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(shape) * scale).astype(np.float16)


def _filled_cache(b, nh, pos, d, bits, gs, seed, garbage_after=True):
    """Cache with random keys/values in slots [0, pos) and, if asked, other random
    values in every later slot (which attention at pos must never read)."""
    S = pos + 3
    cache = layer.KVCache(b, nh, S, d, bits, gs)
    if garbage_after:
        cache.store(_rand16((b, nh, S, d), seed + 50, 3.0), _rand16((b, nh, S, d), seed + 51, 3.0), 0)
    if pos > 0:
        cache.store(_rand16((b, nh, pos, d), seed), _rand16((b, nh, pos, d), seed + 1), 0)
    return cache


def test_decode_attention_pos0_returns_fresh_value():
    """No cached keys: the softmax has the fresh key alone, so o = v_new exactly."""
    b, nh, d = 3, 4, 64
    cache = _filled_cache(b, nh, 0, d, 4, 64, seed=1)
    q, kn, vn = _rand16((b, nh, d), 2), _rand16((b, nh, d), 3), _rand16((b, nh, d), 4)
    o = layer.decode_attention(q, kn, vn, cache, 0)
    assert np.array_equal(o, vn.astype(np.float64))


@pytest.mark.parametrize("pos", [1, 5, 17])
def test_decode_attention_equal_keys_give_mean_of_values(pos):
    """Every cached key and the fresh key are the same exactly representable vector
    (each 64-group holds only 0 and 1, which the 4-bit quantiser reproduces exactly),
    so every score is equal and o is the plain mean of the pos cached values and v_new.
    The values take two levels {a, a + 1} per group (a small integer), also exact."""
    b, nh, d = 2, 3, 128
    rng = np.random.default_rng(pos)
    key = rng.integers(0, 2, size=(b, nh, 1, d)).astype(np.float16)
    keys = np.repeat(key, pos, axis=2)
    base = rng.integers(-2, 3, size=(b, nh, pos, d // 64, 1))
    vals = (base + rng.integers(0, 2, size=(b, nh, pos, d // 64, 64))).reshape(b, nh, pos, d).astype(np.float16)
    cache = layer.KVCache(b, nh, pos + 2, d)
    cache.store(keys, vals, 0)
    kc, vc = cache.load(pos)
    assert np.array_equal(kc, keys.astype(np.float64)) and np.array_equal(vc, vals.astype(np.float64))
    q = _rand16((b, nh, d), 7)
    vn = rng.integers(-3, 4, size=(b, nh, d)).astype(np.float16)
    o = layer.decode_attention(q, key[:, :, 0], vn, cache, pos)
    expect = (vals.astype(np.float64).sum(axis=2) + vn.astype(np.float64)) / (pos + 1)
    assert np.max(np.abs(o - expect)) <= 1e-12 * max(1.0, np.abs(expect).max())


def _slot(codes, meta, d, bits, gs):
    """Dequantised values of one cache slot (one key or value vector), via the codec."""
    return codec.decompress(codes, meta, (d,), num_bits=bits, group_size=gs, group_dim=0).astype(np.float64)


@pytest.mark.parametrize("bits,gs,pos", [(4, 64, 9), (8, 32, 6), (4, 32, 1)])
def test_decode_attention_brute_force(bits, gs, pos):
    """Pure-Python loops: for every (sequence, head) decompress slots 0..pos-1 one by
    one, append the fresh key/value, softmax with the max subtracted, weighted sum.
    Slots >= pos hold other data, so reading one slot too many fails."""
    b, nh, d = 2, 2, 64
    cache = _filled_cache(b, nh, pos, d, bits, gs, seed=10 * pos + bits)
    q, kn, vn = _rand16((b, nh, d), 11, 0.2), _rand16((b, nh, d), 12), _rand16((b, nh, d), 13)
    o = layer.decode_attention(q, kn, vn, cache, pos)
    for bi in range(b):
        for hd in range(nh):
            keys, vals = [], []
            for j in range(pos):
                keys.append(_slot(cache.k_codes[bi, hd, j], cache.k_meta[bi, hd, j], d, bits, gs).tolist())
                vals.append(_slot(cache.v_codes[bi, hd, j], cache.v_meta[bi, hd, j], d, bits, gs).tolist())
            keys.append(kn[bi, hd].astype(np.float64).tolist())
            vals.append(vn[bi, hd].astype(np.float64).tolist())
            qv = q[bi, hd].astype(np.float64).tolist()
            sc = [sum(qv[e] * kk[e] for e in range(d)) for kk in keys]
            m = max(sc)
            ex = [math.exp(c - m) for c in sc]
            z = sum(ex)
            ref = [sum(ex[j] / z * vals[j][e] for j in range(len(keys))) for e in range(d)]
            assert np.allclose(o[bi, hd], ref, rtol=1e-12, atol=1e-12), (bi, hd)


def test_decode_attention_sequences_and_heads_independent():
    """Permuting the batch permutes the result; a head depends on its own slots only."""
    b, nh, d, pos = 3, 2, 64, 4
    cache = _filled_cache(b, nh, pos, d, 4, 64, seed=20, garbage_after=False)
    q, kn, vn = _rand16((b, nh, d), 21), _rand16((b, nh, d), 22), _rand16((b, nh, d), 23)
    o = layer.decode_attention(q, kn, vn, cache, pos)
    perm = [2, 0, 1]
    c2 = layer.KVCache(b, nh, pos + 3, d)
    for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
        getattr(c2, name)[:] = getattr(cache, name)[perm]
    o2 = layer.decode_attention(q[perm], kn[perm], vn[perm], c2, pos)
    assert np.array_equal(o2, o[perm])
    c2.k_codes[:, 1] ^= 0x11                                  # disturb head 1's keys only
    o3 = layer.decode_attention(q[perm], kn[perm], vn[perm], c2, pos)
    assert np.array_equal(o3[:, 0], o2[:, 0]) and not np.array_equal(o3[:, 1], o2[:, 1])


def test_prefill_attention_single_token_is_value():
    """s = 1: each query sees only its own key, so o = v exactly."""
    q, k, v = _rand16((2, 1, 3, 64), 30), _rand16((2, 1, 3, 64), 31), _rand16((2, 1, 3, 64), 32)
    o = layer.prefill_attention(q, k, v)
    assert np.array_equal(o, v.astype(np.float64))


def test_prefill_attention_brute_force_layout():
    """Pure-Python loops over the [batch][seq][heads][head_dim] layout: row i of head h
    attends to keys j <= i of the same head. Heads, tokens and dims all differ in
    count, so a transposed axis fails."""
    b, s, nh, d = 2, 5, 3, 8
    q, k, v = _rand16((b, s, nh, d), 40), _rand16((b, s, nh, d), 41), _rand16((b, s, nh, d), 42)
    o = layer.prefill_attention(q, k, v)
    assert o.shape == (b, s, nh, d)
    qf, kf, vf = (t.astype(np.float64).tolist() for t in (q, k, v))
    for bi in range(b):
        for i in range(s):
            for hd in range(nh):
                sc = [sum(qf[bi][i][hd][e] * kf[bi][j][hd][e] for e in range(d)) for j in range(i + 1)]
                m = max(sc)
                ex = [math.exp(c - m) for c in sc]
                z = sum(ex)
                ref = [sum(ex[j] / z * vf[bi][j][hd][e] for j in range(i + 1)) for e in range(d)]
                assert np.allclose(o[bi, i, hd], ref, rtol=1e-12, atol=1e-12), (bi, i, hd)


def test_prefill_attention_is_causal():
    b, s, nh, d = 1, 6, 2, 16
    q, k, v = _rand16((b, s, nh, d), 50), _rand16((b, s, nh, d), 51), _rand16((b, s, nh, d), 52)
    o = layer.prefill_attention(q, k, v)
    k2, v2 = k.copy(), v.copy()
    k2[:, 3:] = _rand16((b, s - 3, nh, d), 53)
    v2[:, 3:] = _rand16((b, s - 3, nh, d), 54)
    o2 = layer.prefill_attention(q, k2, v2)
    assert np.array_equal(o[:, :3], o2[:, :3]) and not np.array_equal(o[:, 3:], o2[:, 3:])


def test_linear_fp16_weight_blocks_match_dense():
    """The block-wise product on a float16 weight (used for the large layers) equals the
    product on the same weight widened to float64 at once."""
    w = synth.normal_f16((300, 256), 60, 0.02).numpy()
    a = synth.normal_f16((3, 256), 61).numpy().astype(np.float64)
    bias = synth.normal_f16((300,), 62, 0.02).numpy()
    old = layer.ROW_BLOCK_ELEMS
    layer.ROW_BLOCK_ELEMS = 256 * 7                       # 7-row blocks, ragged tail
    try:
        y16 = layer.linear(a, w, bias)
    finally:
        layer.ROW_BLOCK_ELEMS = old
    y64 = a @ w.astype(np.float64).T + bias.astype(np.float64)
    assert np.allclose(y16, y64, rtol=1e-13, atol=1e-13)
