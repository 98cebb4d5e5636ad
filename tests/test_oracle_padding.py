"""Pins of the oracle's left-padding mask (variable prompt lengths).

The pages keep an ``attention_mask`` buffer in the generation loop (source-notes page
«FlexGen» (PtirisNote), "Flex Opt") and pad HELM prompts to ``pad_to_seq_len``
(walkthrough page, section 3.1). Reading: prompts are padded on the left; sequence b's
real tokens start at valid_from[b]; no query attends to a pad key; a pad query (which
has no visible key) gets a zero attention output.

The layer holds no positional term, so a left-padded prompt must give, on its real
rows, exactly what the unpadded prompt gives alone - prefill rows, cache contents and
every later decode step. That relation, a zero-mask identity and the pad-row closed
form pin the masked oracle to the unmasked one (itself pinned elsewhere).
"""
import numpy as np
import pytest

import synth
from oracle import layer


def _params(h=128, ffn=256, seed=3):
    raw = {k: v.numpy() for k, v in synth.layer_params(h, ffn, seed).items()}
    PQ = layer.compress_weights(raw)
    return PQ, layer.dequant_all(PQ)


def _close(a, b, rel=1e-12):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    assert a.shape == b.shape
    assert np.max(np.abs(a - b)) <= rel * max(1.0, np.max(np.abs(b))), np.max(np.abs(a - b))


def test_zero_mask_is_unmasked():
    PQ, W = _params()
    x = synth.activations((2, 6, 128), 1).numpy()
    c1, c2 = layer.KVCache(2, 2, 8, 64), layer.KVCache(2, 2, 8, 64)
    assert np.array_equal(layer.prefill_layer(x, PQ, c1, 2, W=W),
                          layer.prefill_layer(x, PQ, c2, 2, W=W, valid_from=[0, 0]))
    xd = synth.decode_inputs(2, 128, 0, 1).numpy()
    assert np.array_equal(layer.decode_layer(xd, PQ, c1, 6, 2, W=W),
                          layer.decode_layer(xd, PQ, c2, 6, 2, W=W, valid_from=[0, 0]))


@pytest.mark.parametrize("P", [1, 3, 5])
def test_left_padded_prompt_equals_unpadded_prompt(P):
    """Sequence 1 is padded with P tokens (any values); sequence 0 is not. Real rows,
    cache slots and two decode steps match the unpadded run of each sequence alone; pad
    rows are the layer with a zero attention output."""
    h, nh, s = 128, 2, 7
    PQ, W = _params()
    x = synth.activations((2, s, h), 2 + P).numpy()
    vf = [0, P]
    cache = layer.KVCache(2, nh, s + 3, 64)
    out = layer.prefill_layer(x, PQ, cache, nh, W=W, valid_from=vf).astype(np.float64)
    # sequence 1 alone, without its pad tokens
    c1 = layer.KVCache(1, nh, s + 3, 64)
    ref1 = layer.prefill_layer(x[1:2, P:].copy(), PQ, c1, nh, W=W).astype(np.float64)
    _close(out[1, P:], ref1[0])
    # sequence 0 is unaffected by its neighbour's padding
    c0 = layer.KVCache(1, nh, s + 3, 64)
    ref0 = layer.prefill_layer(x[0:1].copy(), PQ, c0, nh, W=W).astype(np.float64)
    _close(out[0], ref0[0])
    # pad rows: zero attention output, then the rest of the block
    pad = layer.mlp_block(x[1:2, :P].astype(np.float64), np.zeros((1, P, h)), PQ, W).astype(np.float16)
    _close(out[1, :P], pad[0].astype(np.float64))
    # the real tokens' cache slots are those of the unpadded run, shifted by P
    assert (cache.k_codes[1, :, P:s] == c1.k_codes[0, :, :s - P]).mean() > 0.999
    assert (cache.v_codes[1, :, P:s] == c1.v_codes[0, :, :s - P]).mean() > 0.999
    # decode steps: padded at pos s + t, unpadded at pos s - P + t, over the same history
    for t in range(2):
        xd = synth.decode_inputs(2, h, t, 40 + P).numpy()
        d = layer.decode_layer(xd, PQ, cache, s + t, nh, W=W, valid_from=vf).astype(np.float64)
        r1 = layer.decode_layer(xd[1:2].copy(), PQ, c1, s - P + t, nh, W=W).astype(np.float64)
        r0 = layer.decode_layer(xd[0:1].copy(), PQ, c0, s + t, nh, W=W).astype(np.float64)
        _close(d[1], r1[0], rel=2e-3)          # caches may differ in a rare fp16 tie of k/v
        _close(d[0], r0[0])


def test_decode_attention_ignores_pad_slots():
    """Slots below valid_from change nothing; the result equals attention over a cache
    that holds only the real slots."""
    b, nh, d, pos, P = 2, 3, 64, 9, 4
    rng = np.random.default_rng(5)
    kh = rng.standard_normal((b, nh, pos, d)).astype(np.float16)
    vh = rng.standard_normal((b, nh, pos, d)).astype(np.float16)
    q, kn, vn = (rng.standard_normal((b, nh, d)).astype(np.float16) for _ in range(3))
    c = layer.KVCache(b, nh, pos + 1, d)
    c.store(kh, vh, 0)
    o = layer.decode_attention(q, kn, vn, c, pos, valid_from=[P, P])
    c2 = layer.KVCache(b, nh, pos + 1, d)
    c2.store((kh * 3).astype(np.float16)[:, :, :P], (vh - 2).astype(np.float16)[:, :, :P], 0)
    c2.store(kh[:, :, P:], vh[:, :, P:], P)
    _close(layer.decode_attention(q, kn, vn, c2, pos, valid_from=[P, P]), o, rel=0)
    c3 = layer.KVCache(b, nh, pos - P + 1, d)
    c3.store(kh[:, :, P:], vh[:, :, P:], 0)
    _close(layer.decode_attention(q, kn, vn, c3, pos - P), o, rel=0)
    # everything padded but the new token: o = v_new
    assert np.array_equal(layer.decode_attention(q, kn, vn, c, pos, valid_from=[pos, pos]), vn.astype(np.float64))


def test_prefill_attention_pad_rows_zero_and_real_rows_trimmed():
    b, s, nh, d, P = 1, 6, 2, 16, 2
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((b, s, nh, d)).astype(np.float16) for _ in range(3))
    o = layer.prefill_attention(q, k, v, valid_from=[P])
    assert np.array_equal(o[:, :P], np.zeros((b, P, nh, d)))
    _close(o[:, P:], layer.prefill_attention(q[:, P:], k[:, P:], v[:, P:]), rel=0)
