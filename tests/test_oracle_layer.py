"""Pins of the oracle OPT layer (prefill ``mha`` and decode ``mha_gen``).

Checks against closed forms (LayerNorm of a +-a row, identity layer, uniform
attention = running mean, one-token prompt), invariants (softmax rows sum to one,
causality, batch independence, head-feature layout), a brute-force triple-loop
layer on tiny sizes, and the decode/prefill relation (a decode step at pos p sees
what prefill row p sees, up to the cache quantisation, whose effect shrinks with
the quantisation step).
"""
import math

import numpy as np
import pytest

from oracle import codec, layer
import synth


def tiny_params(h=128, ffn=256, seed=3):
    raw = {k: v.numpy() for k, v in synth.layer_params(h, ffn, seed).items()}
    return raw


def quantised(raw):
    return layer.compress_weights(raw)


def zero_like_params(raw):
    return {k: np.zeros_like(v) for k, v in raw.items()}


def test_layer_norm_closed_form():
    a = 1.5
    row = np.array([a, -a] * 8, np.float64)
    g = np.linspace(0.5, 2.0, 16)
    b = np.linspace(-1, 1, 16)
    y = layer.layer_norm(row[None], g, b)[0]
    expect = np.array([1, -1] * 8) * a / math.sqrt(a * a + 1e-5) * g + b
    assert np.allclose(y, expect, rtol=0, atol=1e-14)
    # a constant row normalises to beta
    y2 = layer.layer_norm(np.full((1, 16), 7.25), g, b)[0]
    assert np.allclose(y2, b, atol=1e-14)


def test_softmax_rows_sum_to_one_and_causal():
    rng = np.random.default_rng(0)
    q = rng.standard_normal((2, 3, 9, 16))
    k = rng.standard_normal((2, 3, 9, 16))
    p = layer.attention_probs_prefill(q, k)
    assert np.allclose(p.sum(-1), 1.0, atol=1e-12)
    assert np.all(p >= 0)
    assert np.all(p[..., np.triu_indices(9, 1)[0], np.triu_indices(9, 1)[1]] == 0)
    assert np.allclose(p[..., 0, 0], 1.0)


def test_identity_layer():
    """All weights and biases zero: q = k = v = 0, o = 0, f = 0, so out = x."""
    raw = zero_like_params(tiny_params())
    raw["ln1_g"] = np.ones(128, np.float16)
    raw["ln2_g"] = np.ones(128, np.float16)
    PQ = quantised(raw)
    x = synth.activations((2, 5, 128), 7).numpy()
    cache = layer.KVCache(2, 2, 8, 64)
    out = layer.prefill_layer(x, PQ, cache, 2)
    assert np.array_equal(out, x)
    xd = synth.decode_inputs(2, 128, 0, 7).numpy()
    outd = layer.decode_layer(xd, PQ, cache, 5, 2)
    assert np.array_equal(outd, xd)


def _exact_grid_weight(rows, cols, fn):
    """A weight whose entries are exactly representable after 4-bit g64 quantisation:
    every 64-group holds only the values {0, 1}, or only {0}."""
    w = np.zeros((rows, cols), np.float16)
    for r in range(rows):
        for c in range(cols):
            w[r, c] = fn(r, c)
    return w


def test_uniform_attention_is_running_mean_and_head_layout():
    """Wq = Wk = 0 for every head except head 0: heads 1.. attend uniformly, so their
    output is the running mean of v over j <= i. Wv = permutation, Wo = identity,
    FFN zero: out = x + (mixed head outputs)[perm] + b_o + b_fc2. Head 0 differs.
    This fixes the [q; k; v] row order and feature = head * d + j."""
    h, nh, d, s = 128, 2, 64, 6
    raw = zero_like_params(tiny_params())
    raw["ln1_g"] = np.ones(h, np.float16)
    raw["ln2_g"] = np.ones(h, np.float16)
    perm = np.roll(np.arange(h), 5)
    Wq = np.zeros((h, h), np.float16)
    Wk = np.zeros((h, h), np.float16)
    Wq[0:d, 0:d] = np.eye(d, dtype=np.float16)           # head 0 only
    Wk[0:d, 0:d] = np.eye(d, dtype=np.float16)
    Wv = np.eye(h, dtype=np.float16)[perm]                 # v[j] = a[perm[j]]
    raw["w_qkv"] = np.concatenate([Wq, Wk, Wv], 0)
    raw["w_o"] = np.eye(h, dtype=np.float16)
    PQ = quantised(raw)
    # 0/1 matrices are exact after quantisation (min 0, max 1, scale 15, levels k/15)
    W = layer.dequant_all(PQ)
    assert np.array_equal(W["w_qkv"], raw["w_qkv"].astype(np.float64))
    x = synth.activations((1, s, h), 9).numpy()
    cache = layer.KVCache(1, nh, 8, d)
    out = layer.prefill_layer(x, PQ, cache, nh).astype(np.float64)
    a = layer.layer_norm(x.astype(np.float64), raw["ln1_g"], raw["ln1_b"])[0]   # [s][h]
    v = a[:, perm]
    running = np.cumsum(v, 0) / np.arange(1, s + 1)[:, None]
    expect = x[0].astype(np.float64) + running
    tol = 2.0 ** -10 * np.abs(expect) + 1e-6
    assert np.all(np.abs(out[0][:, d:] - expect[:, d:]) <= tol[:, d:])   # heads >= 1
    # head 0 has real attention: later rows differ from the running mean
    assert np.max(np.abs(out[0][2:, :d] - expect[2:, :d])) > 1e-3


def test_one_token_prompt_attends_to_itself():
    """s = 1: the softmax has one entry, so o = v exactly (per head)."""
    raw = tiny_params()
    PQ = quantised(raw)
    W = layer.dequant_all(PQ)
    x = synth.activations((3, 1, 128), 10).numpy()
    q, k, v = layer.qkv_projection(x.astype(np.float64), PQ, W["w_qkv"], 2)
    p = layer.attention_probs_prefill(q, k)
    assert np.array_equal(p, np.ones_like(p))
    cache = layer.KVCache(3, 2, 4, 64)
    out = layer.prefill_layer(x, PQ, cache, 2)
    o = np.moveaxis(v, 1, 2).reshape(3, 1, 128)
    expect = layer.mlp_block(x.astype(np.float64), o, PQ, W).astype(np.float16)
    assert np.array_equal(out, expect)


def test_causality():
    raw = tiny_params()
    PQ = quantised(raw)
    x = synth.activations((2, 7, 128), 11).numpy()
    out1 = layer.prefill_layer(x, PQ, layer.KVCache(2, 2, 8, 64), 2)
    x2 = x.copy()
    x2[:, 4:] = synth.activations((2, 3, 128), 12).numpy()
    out2 = layer.prefill_layer(x2, PQ, layer.KVCache(2, 2, 8, 64), 2)
    assert np.array_equal(out1[:, :4], out2[:, :4])
    assert not np.array_equal(out1[:, 4:], out2[:, 4:])


def test_batch_independence():
    raw = tiny_params()
    PQ = quantised(raw)
    x = synth.activations((3, 5, 128), 13).numpy()
    out = layer.prefill_layer(x, PQ, layer.KVCache(3, 2, 8, 64), 2)
    out_rev = layer.prefill_layer(x[::-1].copy(), PQ, layer.KVCache(3, 2, 8, 64), 2)
    assert np.array_equal(out, out_rev[::-1])
    one = layer.prefill_layer(x[1:2].copy(), PQ, layer.KVCache(1, 2, 8, 64), 2)
    assert np.array_equal(one[0], out[1])


def _brute_layer(x, W, P, nh, cache_k=None, cache_v=None):
    """Triple-loop statement of the layer for tiny sizes (python floats).

    x: list [s][h] (one sequence); cache_k/v: optional list [nh][p][d] of already
    dequantised past keys/values, attended before the s fresh tokens (decode when
    s = 1)."""
    s, h = len(x), len(x[0])
    d = h // nh

    def ln(row, g, b):
        mu = sum(row) / h
        var = sum((r - mu) ** 2 for r in row) / h
        return [(row[i] - mu) / math.sqrt(var + 1e-5) * g[i] + b[i] for i in range(h)]

    def lin(row, w, b):
        return [sum(w[o][i] * row[i] for i in range(len(row))) + b[o] for o in range(len(w))]

    past = 0 if cache_k is None else len(cache_k[0])
    qs, ks, vs = [], [], []
    for t in range(s):
        a = ln(x[t], P["ln1_g"], P["ln1_b"])
        qkv = lin(a, W["w_qkv"], P["b_qkv"])
        qs.append([qkv[i] / math.sqrt(d) for i in range(h)])
        ks.append(qkv[h:2 * h])
        vs.append(qkv[2 * h:])
    outs = []
    for t in range(s):
        o = [0.0] * h
        for hd in range(nh):
            keys, vals = [], []
            for j in range(past):
                keys.append(cache_k[hd][j])
                vals.append(cache_v[hd][j])
            for j in range(t + 1):
                keys.append(ks[j][hd * d:(hd + 1) * d])
                vals.append(vs[j][hd * d:(hd + 1) * d])
            sc = [sum(qs[t][hd * d + e] * kk[e] for e in range(d)) for kk in keys]
            m = max(sc)
            ex = [math.exp(c - m) for c in sc]
            z = sum(ex)
            for e in range(d):
                o[hd * d + e] = sum(ex[j] / z * vals[j][e] for j in range(len(keys)))
        h1 = [x[t][i] + v for i, v in enumerate(lin(o, W["w_o"], P["b_o"]))]
        a2 = ln(h1, P["ln2_g"], P["ln2_b"])
        f = [max(0.0, v) for v in lin(a2, W["w_fc1"], P["b_fc1"])]
        outs.append([h1[i] + v for i, v in enumerate(lin(f, W["w_fc2"], P["b_fc2"]))])
    return outs, ks, vs


def test_brute_force_tiny_layer_prefill_and_decode():
    h, nh, d, ffn, b, s = 128, 2, 64, 256, 2, 3
    raw = tiny_params(h, ffn, seed=21)
    PQ = quantised(raw)
    W = layer.dequant_all(PQ)
    Wl = {k: v.tolist() for k, v in W.items()}
    Pl = {k: raw[k].astype(np.float64).tolist() for k in
          ("ln1_g", "ln1_b", "ln2_g", "ln2_b", "b_qkv", "b_o", "b_fc1", "b_fc2")}
    x = synth.activations((b, s, h), 22).numpy()
    cache = layer.KVCache(b, nh, 8, d)
    out = layer.prefill_layer(x, PQ, cache, nh).astype(np.float64)
    for bi in range(b):
        ref, _, _ = _brute_layer(x[bi].astype(np.float64).tolist(), Wl, Pl, nh)
        ref = np.array(ref)
        assert np.all(np.abs(out[bi] - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-9)
    # one decode step at pos s over the cache the prefill wrote
    xd = synth.decode_inputs(b, h, 0, 22).numpy()
    kc, vc = cache.load(s)
    outd = layer.decode_layer(xd, PQ, cache, s, nh).astype(np.float64)
    for bi in range(b):
        ref, _, _ = _brute_layer([xd[bi].astype(np.float64).tolist()], Wl, Pl, nh,
                                 kc[bi].tolist(), vc[bi].tolist())
        ref = np.array(ref[0])
        assert np.all(np.abs(outd[bi] - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-9)


def test_prefill_stores_quantised_fp16_kv():
    """Prefill writes slots [0, s): their dequantised keys are within the quantiser's
    error bound of the layer's own keys; slots >= s stay untouched."""
    raw = tiny_params()
    PQ = quantised(raw)
    W = layer.dequant_all(PQ)
    x = synth.activations((2, 5, 128), 23).numpy()
    cache = layer.KVCache(2, 2, 8, 64)
    layer.prefill_layer(x, PQ, cache, 2)
    _, k, v = layer.qkv_projection(x.astype(np.float64), PQ, W["w_qkv"], 2)
    kc, vc = cache.load(5)
    r = k.max(-1) - k.min(-1)
    assert np.all(np.abs(kc - k) <= (r / 30 * 1.001 + 2.0 ** -10 * np.abs(k).max(-1) + 1e-6)[..., None])
    assert np.all(cache.k_codes[:, :, 5:] == 0) and np.all(cache.k_meta[:, :, 5:] == 0)


@pytest.mark.parametrize("p", [1, 6])
def test_decode_matches_prefill_row_up_to_cache_quantisation(p):
    """Decode at pos p over the cache of tokens [0, p) sees what prefill row p sees, except
    that past keys/values went through the cache quantiser. The gap must shrink about
    16x from a 4-bit to an 8-bit cache (step ratio 255/15 = 17)."""
    raw = tiny_params()
    x = synth.activations((2, p + 1, 128), 24).numpy()
    gaps = {}
    for bits in (4, 8):
        PQ = quantised(raw)
        full = layer.prefill_layer(x, PQ, layer.KVCache(2, 2, 8, 64, num_bits=bits), 2).astype(np.float64)
        cache = layer.KVCache(2, 2, 8, 64, num_bits=bits)
        layer.prefill_layer(x[:, :p].copy(), PQ, cache, 2)
        dec = layer.decode_layer(x[:, p].copy(), PQ, cache, p, 2).astype(np.float64)
        gaps[bits] = np.max(np.abs(dec - full[:, p]))
    scale = np.max(np.abs(x))
    assert gaps[4] < 0.05 * scale
    assert gaps[8] < gaps[4] / 4 + 2e-3
