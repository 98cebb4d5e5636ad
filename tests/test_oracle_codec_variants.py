"""Pins of the oracle codec's variants: the symmetric (absmax) form, 3-bit codes and
zero-padded partial groups. Readings of what the pages only name (the walkthrough page,
section 6.3: the symmetric flag and num_groups groups along group_dim; the hub page:
int3/int4 group-wise quantisation); each is pinned by hand-worked examples
(tests/golden/codec_variant_examples.json) and by invariants that a wrong sign, offset,
bit order or padding position would break."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import codec


def _examples(golden_dir):
    with open(os.path.join(golden_dir, "codec_variant_examples.json")) as f:
        return {e["name"]: e for e in json.load(f)["examples"]}


@pytest.mark.parametrize("name", ["F_symmetric_4bit", "G_three_bit", "H_partial_group"])
def test_variant_worked_examples(golden_dir, name):
    e = _examples(golden_dir)[name]
    x = np.array(e["x"], np.float16).reshape(e["shape"])
    kw = dict(num_bits=e["num_bits"], group_size=e["group_size"], group_dim=e["group_dim"], symmetric=e["symmetric"])
    c, m = codec.compress(x, **kw)
    assert c.ravel().tolist() == e["codes"]
    assert m.reshape(-1, 2).astype(np.float64).tolist() == e["meta"]
    y = codec.decompress(c, m, x.shape, **kw)
    assert y.shape == x.shape
    if "decompressed" in e:
        assert y.astype(np.float64).tolist() == [float(v) for v in e["decompressed"]]
    else:                                                  # H: the whole first group is exact
        assert np.array_equal(y[:32], x[:32])


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_symmetric_sign_mirror_and_bound(bits):
    """codes(-x) = 2B - codes(x) with the same scale (rint is odd), and |x^ - x| stays
    within half a step of the absmax grid (plus fp16 slack)."""
    x = synth.codec_tensor((32, 256), 1, 64, seed=bits).numpy()
    B = (1 << (bits - 1)) - 1
    c, m = codec.compress(x, bits, 64, 1, symmetric=True)
    cn, mn = codec.compress((-x).astype(np.float16), bits, 64, 1, symmetric=True)
    assert np.array_equal(m, mn)
    q = codec.unpack(c.reshape(32, 4, -1), bits).astype(int)
    qn = codec.unpack(cn.reshape(32, 4, -1), bits).astype(int)
    assert np.array_equal(qn, 2 * B - q)
    y = codec.decompress(c, m, x.shape, bits, 64, 1, symmetric=True).astype(np.float64)
    a = np.abs(x.astype(np.float64)).reshape(32, 4, 64).max(-1)
    s = m[..., 1].astype(np.float64)
    ok = (s > 0) & (s < 65504)
    err = np.abs(y - x).reshape(32, 4, 64).max(-1)
    bound = a / (2 * B) * (1 + 2.0 ** -9) + 2.0 ** -10 * a + 1e-7
    assert np.all(err[ok] <= bound[ok])


def test_symmetric_zero_group():
    x = np.zeros(64, np.float16)
    c, m = codec.compress(x, 4, 64, 0, symmetric=True)
    assert m.tolist() == [[0.0, 0.0]]
    assert np.all(codec.unpack(c.reshape(1, -1), 4) == 7)
    assert np.array_equal(codec.decompress(c, m, x.shape, 4, 64, 0, symmetric=True), x)


def test_three_bit_pack_round_trip_and_nearest_level():
    rng = np.random.default_rng(0)
    q = rng.integers(0, 8, size=(5, 3, 64)).astype(np.uint8)
    assert np.array_equal(codec.unpack(codec.pack(q, 3), 3), q)
    assert codec.pack(q, 3).shape == (5, 3, 24)
    # each code is the nearest level of (x - min) * scale under the stored fp16 scale
    x = np.round(rng.standard_normal((4, 64)) * 8).astype(np.float16) / np.float16(4)
    c, m = codec.compress(x, 3, 64, 1)
    codes = codec.unpack(c.reshape(4, 1, 24), 3)[:, 0]
    for r in range(4):
        mn, s = Fraction(float(m[r, 0, 0])), Fraction(float(m[r, 0, 1]))
        for j in range(64):
            t = (Fraction(float(x[r, j])) - mn) * s
            best = min(range(8), key=lambda k: (abs(t - k), k % 2))      # nearest, ties to even
            if abs(t - best) != abs(t - int(codes[r, j])):
                raise AssertionError((r, j, float(t), best, int(codes[r, j])))


@pytest.mark.parametrize("shape,gd", [((100,), 0), ((3, 70), 1), ((150, 5), 0), ((2, 33, 4), 1)])
def test_partial_group_is_zero_padded(shape, gd):
    """A dim that is not a multiple of the group: the same codes and metadata as the
    explicitly zero-padded tensor, and decompression returns the original extent."""
    x = synth.codec_tensor(tuple(d if i != gd else -(-d // 32) * 32 for i, d in enumerate(shape)), gd, 32, 4).numpy()
    sl = tuple(slice(0, d) for d in shape)
    xs = np.ascontiguousarray(x[sl])
    xp = np.zeros_like(x)
    xp[sl] = xs
    c, m = codec.compress(xs, 4, 32, gd)
    cp, mp = codec.compress(xp, 4, 32, gd)
    assert np.array_equal(c, cp) and np.array_equal(m.view(np.uint16), mp.view(np.uint16))
    y = codec.decompress(c, m, xs.shape, 4, 32, gd)
    assert y.shape == xs.shape
    assert np.array_equal(y, codec.decompress(cp, mp, xp.shape, 4, 32, gd)[sl])
    assert codec.num_groups(xs.shape, 32, gd) == -(-shape[gd] // 32)
