"""Pins of the oracle's whole-model pieces (oracle.model): the input embedding, the
output head and the greedy choice, and a tiny end-to-end generation step checked
against pure-Python loops."""
import math

import numpy as np

import synth
from oracle import codec, layer, model


def test_embed_is_dequantised_row_plus_position():
    """Token rows whose 64-groups hold only {0, 1} are exact after quantisation, so the
    embedding is the plain sum of the raw table row and the position row."""
    V, h = 10, 128
    rng = np.random.default_rng(0)
    E = rng.integers(0, 2, size=(V, h)).astype(np.float16)
    P = (rng.integers(-4, 5, size=(6, h)) / 4).astype(np.float16)
    E_hat = model.dequant_table(model.compress_table(E))
    assert np.array_equal(E_hat, E)
    x = model.embed([3, 0, 9], [5, 0, 2], E_hat, P)
    assert np.array_equal(x, (E[[3, 0, 9]].astype(np.float64) + P[[5, 0, 2]]).astype(np.float16))


def test_head_logits_brute_force_and_greedy_ties():
    V, h = 7, 64
    rng = np.random.default_rng(1)
    E_hat = rng.standard_normal((V, h)).astype(np.float16)
    g = (1 + 0.1 * rng.standard_normal(h)).astype(np.float16)
    b = (0.1 * rng.standard_normal(h)).astype(np.float16)
    hh = rng.standard_normal((2, h)).astype(np.float16)
    lg = model.logits(hh, g, b, E_hat)
    for r in range(2):
        row = hh[r].astype(np.float64).tolist()
        mu = sum(row) / h
        var = sum((v - mu) ** 2 for v in row) / h
        a = [(row[i] - mu) / math.sqrt(var + 1e-5) * float(g[i]) + float(b[i]) for i in range(h)]
        for v in range(V):
            ref = sum(a[i] * float(E_hat[v, i]) for i in range(h))
            assert abs(lg[r, v] - ref) <= 1e-12 * max(1.0, abs(ref))
    assert model.greedy(np.array([[1.0, 3.0, 3.0, -1.0], [0.0, 0.0, 0.0, 0.0]])).tolist() == [1, 0]


def test_tiny_model_step_matches_direct_composition():
    """One layer, prompt of 3 tokens, one decode step: the model's logits equal the
    composition of the independently pinned pieces (embedding, oracle layer, head)."""
    h, nh, ffn, V = 128, 2, 256, 50
    raw = {k: v.numpy() for k, v in synth.layer_params(h, ffn, 5).items()}
    E = synth.normal_f16((V, h), 6, 0.02).numpy()
    P = synth.normal_f16((8, h), 7, 0.02).numpy()
    g = synth.normal_f16((h,), 8, 0.02, mean=1.0).numpy()
    bb = synth.normal_f16((h,), 9, 0.02).numpy()
    m = model.Model([raw], nh, E, P, g, bb)
    prompt = np.array([[4, 17, 2], [0, 49, 33]])
    caches = m.new_caches(2, 8, 64)
    lg = m.prefill(prompt, caches)
    PQ = layer.compress_weights(raw)
    c2 = layer.KVCache(2, nh, 8, 64)
    E_hat = model.dequant_table(model.compress_table(E))
    x = model.embed(prompt.reshape(-1), [0, 1, 2, 0, 1, 2], E_hat, P).reshape(2, 3, h)
    y = layer.prefill_layer(x, PQ, c2, nh)
    assert np.allclose(lg, model.logits(y[:, -1], g, bb, E_hat), rtol=0, atol=1e-12)
    nxt = model.greedy(lg)
    lg2 = m.decode(nxt, 3, caches)
    y2 = layer.decode_layer(model.embed(nxt, [3, 3], E_hat, P), PQ, c2, 3, nh)
    assert np.allclose(lg2, model.logits(y2, g, bb, E_hat), rtol=0, atol=1e-12)
