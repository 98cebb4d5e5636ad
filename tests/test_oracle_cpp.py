"""Pins of the plain C++17 fp32 oracle (``oracle/cpp/flexq_oracle.cpp``).

Its fp16 conversions are checked against numpy's IEEE conversions (every fp16 value,
every rounding midpoint and its neighbours, random bit patterns); its codec against the
hand-worked golden examples and bit for bit against the numpy oracle; its layer against
closed forms (identity layer, uniform attention = running mean), invariants (causality,
batch and thread-count independence, decode = prefill row up to the cache
quantisation) and against the independently written numpy fp64 oracle.
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle import codec, cpp, layer


def test_half_to_float_every_value():
    h = np.arange(65536, dtype=np.uint16)
    ref = h.view(np.float16).astype(np.float32)
    got = np.array([cpp.half_to_float(int(i)) for i in range(65536)], np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_float_to_half_midpoints_neighbours_and_random():
    fin = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = ((fin[:-1] + fin[1:]) / 2).astype(np.float32)          # exact in fp32: ties
    around = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
                             np.float32([65504, 65519.99, 65520, 65536, 1e9, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
                                         2.0 ** -14, 0.0])])
    rng = np.random.default_rng(0)
    rnd = rng.integers(0, 2 ** 32, size=400000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    for x in (around, -around, rnd):
        ref = x.astype(np.float16).view(np.uint16)
        assert np.array_equal(cpp.float_to_half_array(x), ref)


def test_codec_golden_examples(golden_dir):
    with open(os.path.join(golden_dir, "codec_worked_examples.json")) as f:
        ex = json.load(f)["examples"]
    by = {e["name"]: e for e in ex}
    for e in ex:
        if "columns" in e:                                  # the strided example: columns of others
            cols = [by[c]["x"] if isinstance(c, str) else [c] * 32 for c in e["columns"]]
            x = np.array(cols, np.float16).T.copy()
            c, m = cpp.compress(x, e["num_bits"], e["group_size"], e["group_dim"])
            assert c.T.tolist() == e["codes_columns"] and m.astype(np.float64).tolist() == e["meta"]
            continue
        x = np.array(e["x"], np.float16).reshape(e["shape"])
        c, m = cpp.compress(x, e["num_bits"], e["group_size"], e["group_dim"])
        assert c.ravel().tolist() == e["codes"], e["name"]
        assert np.allclose(m.reshape(-1, 2).astype(np.float64), np.array(e["meta"]), rtol=0, atol=0), e["name"]
        if "decompressed" in e:
            y = cpp.decompress(c, m, x.shape, e["num_bits"], e["group_size"], e["group_dim"])
            assert y.astype(np.float64).ravel().tolist() == [float(v) for v in e["decompressed"]], e["name"]


@pytest.mark.parametrize("shape,gd", [((48, 256), 1), ((256, 40), 0), ((4, 128, 3), 1), ((2, 3, 5, 128), 3),
                                      ((2, 64, 2, 3), 1)])
@pytest.mark.parametrize("bits,gs", [(4, 32), (4, 64), (4, 128), (8, 32), (8, 64), (8, 128)])
def test_codec_matches_numpy_oracle_bit_for_bit(shape, gd, bits, gs):
    if shape[gd] % gs:
        pytest.skip("group does not divide")
    x = synth.codec_tensor(shape, gd, gs, seed=len(shape) * 10 + bits + gs).numpy()
    x.reshape(-1)[:7] = np.float16([3e-5, 3.01e-5, 3.02e-5, 0, -0.0, 0, -0.0])  # tiny ranges, signed zeros
    c1, m1 = codec.compress(x, bits, gs, gd)
    c2, m2 = cpp.compress(x, bits, gs, gd, nthreads=3)
    assert np.array_equal(c1, c2)
    assert np.array_equal(m1.view(np.uint16), m2.view(np.uint16))
    y1 = codec.decompress(c1, m1, shape, bits, gs, gd)
    y2 = cpp.decompress(c2, m2, shape, bits, gs, gd, nthreads=2)
    assert np.array_equal(y1.view(np.uint16), y2.view(np.uint16))


def _zero_params(h, ffn):
    raw = {k: np.zeros_like(v.numpy()) for k, v in synth.layer_params(h, ffn, 1).items()}
    raw["ln1_g"] = np.ones(h, np.float16)
    raw["ln2_g"] = np.ones(h, np.float16)
    return raw


def test_identity_layer():
    h, ffn, nh = 128, 256, 2
    L = cpp.Layer(_zero_params(h, ffn), nh)
    x = synth.activations((2, 5, h), 3).numpy()
    cache = cpp.KVCache(2, nh, 8, 64)
    assert np.array_equal(cpp.prefill_layer(x, L, cache), x)
    xd = synth.decode_inputs(2, h, 0, 3).numpy()
    assert np.array_equal(cpp.decode_layer(xd, L, cache, 5), xd)


def test_uniform_attention_is_running_mean():
    """Wq = Wk = 0 except head 0: heads 1.. attend uniformly, so their output is the
    running mean of v over j <= i; Wv = a permutation, Wo = identity, FFN zero."""
    h, nh, d, s, ffn = 128, 2, 64, 6, 256
    raw = _zero_params(h, ffn)
    perm = np.roll(np.arange(h), 5)
    Wq = np.zeros((h, h), np.float16)
    Wk = np.zeros((h, h), np.float16)
    Wq[0:d, 0:d] = np.eye(d, dtype=np.float16)
    Wk[0:d, 0:d] = np.eye(d, dtype=np.float16)
    raw["w_qkv"] = np.concatenate([Wq, Wk, np.eye(h, dtype=np.float16)[perm]], 0)
    raw["w_o"] = np.eye(h, dtype=np.float16)
    L = cpp.Layer(raw, nh)
    x = synth.activations((1, s, h), 9).numpy()
    out = cpp.prefill_layer(x, L, cpp.KVCache(1, nh, 8, d)).astype(np.float64)
    a = layer.layer_norm(x.astype(np.float64), raw["ln1_g"], raw["ln1_b"])[0]
    running = np.cumsum(a[:, perm], 0) / np.arange(1, s + 1)[:, None]
    expect = x[0].astype(np.float64) + running
    tol = 2.0 ** -10 * np.abs(expect) + 1e-5
    assert np.all(np.abs(out[0][:, d:] - expect[:, d:]) <= tol[:, d:])
    assert np.max(np.abs(out[0][2:, :d] - expect[2:, :d])) > 1e-3


def _small_layer(h=256, nh=4, ffn=512, seed=5):
    return {k: v.numpy() for k, v in synth.layer_params(h, ffn, seed).items()}


def test_causality_batch_and_thread_independence():
    h, nh = 256, 4
    raw = _small_layer(h, nh)
    L = cpp.Layer(raw, nh)
    x = synth.activations((3, 7, h), 11).numpy()
    out = cpp.prefill_layer(x, L, cpp.KVCache(3, nh, 8, 64), nthreads=1)
    assert np.array_equal(out, cpp.prefill_layer(x, L, cpp.KVCache(3, nh, 8, 64), nthreads=5))
    x2 = x.copy()
    x2[:, 4:] = synth.activations((3, 3, h), 12).numpy()
    out2 = cpp.prefill_layer(x2, L, cpp.KVCache(3, nh, 8, 64))
    assert np.array_equal(out[:, :4], out2[:, :4]) and not np.array_equal(out[:, 4:], out2[:, 4:])
    one = cpp.prefill_layer(x[1:2].copy(), L, cpp.KVCache(1, nh, 8, 64))
    assert np.array_equal(one[0], out[1])


@pytest.mark.parametrize("bits", [4, 8])
def test_layer_matches_numpy_fp64_oracle(bits):
    """Prefill of 9 tokens, then two decode steps, each oracle with its own cache: the
    fp32 and fp64 statements agree to well inside the layer tolerance, and the caches
    they write agree except where fp32 and fp64 keys round to different fp16 values."""
    h, nh, ffn, b, s = 256, 4, 512, 2, 9
    raw = _small_layer(h, nh, ffn)
    PQ = layer.compress_weights(raw)
    W = layer.dequant_all(PQ)
    L = cpp.Layer(raw, nh)
    oc = layer.KVCache(b, nh, s + 3, 64, bits)
    cc = cpp.KVCache(b, nh, s + 3, 64, bits)
    x = synth.activations((b, s, h), 7).numpy()
    r64 = layer.prefill_layer(x, PQ, oc, nh, W=W).astype(np.float64)
    r32 = cpp.prefill_layer(x, L, cc).astype(np.float64)
    assert np.max(np.abs(r64 - r32)) <= 1e-3 * np.max(np.abs(r64)) + 2e-3
    assert (oc.k_codes == cc.k_codes).mean() > 0.99 and (oc.v_codes == cc.v_codes).mean() > 0.99
    for t in range(2):
        xd = synth.decode_inputs(b, h, t, 7).numpy()
        d64 = layer.decode_layer(xd, PQ, oc, s + t, nh, W=W).astype(np.float64)
        d32 = cpp.decode_layer(xd, L, cc, s + t).astype(np.float64)
        assert np.max(np.abs(d64 - d32)) <= 1e-3 * np.max(np.abs(d64)) + 2e-3


def test_decode_attention_closed_forms_and_numpy_agreement():
    b, nh, d, pos = 2, 3, 128, 11
    rng = np.random.default_rng(4)
    # pos 0: o = v_new exactly
    c0 = cpp.KVCache(b, nh, 4, d)
    q, kn, vn = (rng.standard_normal((b, nh, d)).astype(np.float16) for _ in range(3))
    assert np.array_equal(cpp.decode_attention(q, kn, vn, c0, 0), vn.astype(np.float32))
    # random cache: agrees with the numpy oracle's decode_attention
    kh = rng.standard_normal((b, nh, pos, d)).astype(np.float16)
    vh = rng.standard_normal((b, nh, pos, d)).astype(np.float16)
    oc = layer.KVCache(b, nh, pos + 2, d)
    oc.store(kh, vh, 0)
    cc = cpp.KVCache(b, nh, pos + 2, d)
    for name in ("k_codes", "v_codes", "k_meta", "v_meta"):
        getattr(cc, name)[:] = getattr(oc, name)
    q = (q.astype(np.float32) * 0.09).astype(np.float16)
    o32 = cpp.decode_attention(q, kn, vn, cc, pos).astype(np.float64)
    o64 = layer.decode_attention(q, kn, vn, oc, pos)
    assert np.max(np.abs(o32 - o64)) <= 1e-5 * max(1.0, np.abs(o64).max())
