"""Pins of the oracle quantiser against what the pages and the mathematics fix.

Sources: the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3 (configuration, packed shape, fp16
scale, "about 70% less weight memory"); the min/max formula of the method. None of
these tests re-types the oracle's own formula: they check hand-worked values,
closed forms, bounds, exact-rational brute force and layout invariants.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import codec
import synth


def _load_golden(golden_dir):
    with open(os.path.join(golden_dir, "codec_worked_examples.json")) as f:
        return json.load(f)


def _by_name(gold):
    return {e["name"]: e for e in gold["examples"]}


@pytest.mark.parametrize("name", ["A_integer_levels", "B_round_half_even", "C_stored_fp16_scale",
                                  "E_eight_bit"])
def test_worked_examples_1d(golden_dir, name):
    ex = _by_name(_load_golden(golden_dir))[name]
    x = np.array(ex["x"], dtype=np.float16)
    codes, meta = codec.compress(x, ex["num_bits"], ex["group_size"], ex["group_dim"])
    assert codes.dtype == np.uint8
    assert codes.tolist() == ex["codes"]
    assert meta.astype(np.float64).tolist() == ex["meta"]
    if "decompressed" in ex:
        y = codec.decompress(codes, meta, x.shape, ex["num_bits"], ex["group_size"], ex["group_dim"])
        assert y.astype(np.float64).tolist() == [float(v) for v in ex["decompressed"]]


def test_worked_example_strided(golden_dir):
    gold = _by_name(_load_golden(golden_dir))
    ex = gold["D_strided_group_dim0"]
    cols = []
    for c in ex["columns"]:
        cols.append(gold[c]["x"] if isinstance(c, str) else [c] * 32)
    x = np.array(cols, dtype=np.float16).T.copy()
    assert x.shape == tuple(ex["shape"])
    codes, meta = codec.compress(x, ex["num_bits"], ex["group_size"], ex["group_dim"])
    assert codes.shape == (16, 3)
    assert codes.T.tolist() == ex["codes_columns"]
    assert meta.astype(np.float64).tolist() == ex["meta"]
    y = codec.decompress(codes, meta, x.shape, 4, 32, 0)
    assert np.all(y[:, 2] == np.float16(3.0))
    assert np.array_equal(y[:, 0], x[:, 0])


def test_size_ratio_matches_pages(golden_dir):
    sr = _load_golden(golden_dir)["size_ratio"]
    shape = (1024, 4096)
    ratio = codec.compressed_bytes(shape, 4, 64) / (2 * np.prod(shape))
    assert ratio == sr["ratio"]
    assert abs((1 - ratio) - sr["pages_saving_approx"]) < 0.03
    x = np.zeros((64, 128), np.float16)
    c, m = codec.compress(x, 4, 64, 1)
    assert c.nbytes + m.nbytes == int(sr["ratio"] * x.nbytes)


@pytest.mark.parametrize("shape,gd,gs,bits", [
    ((4, 256), 1, 64, 4), ((256, 4), 0, 64, 4), ((2, 3, 128), 2, 32, 4),
    ((2, 128, 3), 1, 128, 8), ((3, 2, 4, 64), 3, 64, 4), ((64, 2, 2, 2), 0, 32, 8)])
def test_packed_shape_formula(shape, gd, gs, bits):
    # pages: data_shape = shape[:group_dim] + (num_groups * (group_size // 2),) + shape[group_dim+1:]
    x = np.zeros(shape, np.float16)
    c, m = codec.compress(x, bits, gs, gd)
    ng = shape[gd] // gs
    per = gs // 2 if bits == 4 else gs
    assert c.shape == shape[:gd] + (ng * per,) + shape[gd + 1:]
    assert m.shape == shape[:gd] + (ng,) + shape[gd + 1:] + (2,)
    assert m.dtype == np.float16


def _sweep_tensor(shape, gd, gs, seed):
    return synth.codec_tensor(shape, gd, gs, seed).numpy()


CASES = [((64, 512), 1, 64, 4), ((64, 512), 1, 32, 4), ((64, 512), 1, 128, 4),
         ((64, 512), 1, 64, 8), ((512, 48), 0, 64, 4), ((256, 40), 0, 128, 8),
         ((3, 4, 16, 128), 3, 64, 4), ((2, 128, 5), 1, 32, 4)]


@pytest.mark.parametrize("shape,gd,gs,bits", CASES)
def test_error_bound(shape, gd, gs, bits):
    """|x^ - x| <= range/(2(2^b-1)) up to the fp16 rounding of the scale and of x^.

    Derivation: levels are k/s with s = fp16(B/r) = (B/r)(1+d), |d| <= 2^-11; the
    code is the integer nearest t = (x-min)s (t never exceeds B + 1/2), so
    |x - min - q/s| <= 1/(2s) <= r/(2B)(1+2^-10). Saturated scales (r < B/65504)
    give levels 1/65504 apart instead. Rebuilding adds two fp32 roundings and one
    fp16 rounding (half an ulp: 2^-11 relative, 2^-25 absolute below 2^-14)."""
    x = _sweep_tensor(shape, gd, gs, seed=11)
    c, m = codec.compress(x, bits, gs, gd)
    y = codec.decompress(c, m, x.shape, bits, gs, gd)
    B = (1 << bits) - 1
    xg = np.moveaxis(x.astype(np.float64), gd, -1).reshape(-1, gs)
    yg = np.moveaxis(y.astype(np.float64), gd, -1).reshape(-1, gs)
    r = xg.max(1) - xg.min(1)
    quant = np.maximum(r / (2 * B) * (1 + 2.0 ** -10), 0.5 / 65504 * (1 + 2.0 ** -10))
    quant = np.where(r == 0, 0.0, quant)
    bound = quant[:, None] + 2.0 ** -11 * np.abs(yg) + 2.0 ** -22 * (np.abs(xg.min(1)) + r)[:, None] + 2.0 ** -25
    assert np.all(np.abs(yg - xg) <= bound)


@pytest.mark.parametrize("shape,gd,gs,bits", CASES)
def test_constant_groups_round_trip_exactly(shape, gd, gs, bits):
    x = _sweep_tensor(shape, gd, gs, seed=12)
    c, m = codec.compress(x, bits, gs, gd)
    y = codec.decompress(c, m, x.shape, bits, gs, gd)
    xg = np.moveaxis(x, gd, -1).reshape(-1, gs)
    yg = np.moveaxis(y, gd, -1).reshape(-1, gs)
    const = (xg == xg[:, :1]).all(1)
    assert const.sum() >= 1          # the sweep always plants an all-zero group
    assert np.array_equal(yg[const], xg[const])
    scales = np.moveaxis(m[..., 1], gd, -1).reshape(-1)
    assert np.all(scales[const] == 0)


@pytest.mark.parametrize("shape,gd,gs,bits", CASES)
def test_code_range_and_extremes(shape, gd, gs, bits):
    """Codes lie in [0, 2^b-1]; the group minimum maps to 0, the maximum to 2^b-1."""
    x = _sweep_tensor(shape, gd, gs, seed=13)
    c, m = codec.compress(x, bits, gs, gd)
    B = (1 << bits) - 1
    cm = np.moveaxis(c, gd, -1)
    if bits == 4:
        q = np.empty(cm.shape[:-1] + (cm.shape[-1] * 2,), np.int64)
        q[..., 0::2] = cm & 15          # low nibble = even element (pinned by example A)
        q[..., 1::2] = cm >> 4
    else:
        q = cm.astype(np.int64)
    qg = q.reshape(-1, gs)
    xg = np.moveaxis(x, gd, -1).reshape(-1, gs).astype(np.float32)
    assert qg.min() >= 0 and qg.max() <= B
    nonconst = xg.max(1) > xg.min(1)
    s16 = np.moveaxis(m[..., 1], gd, -1).reshape(-1)
    unsat = nonconst & (s16 < np.float16(65504))
    rows = np.nonzero(unsat)[0]
    assert np.all(qg[rows, xg[rows].argmin(1)] == 0)
    assert np.all(qg[rows, xg[rows].argmax(1)] == B)
    # the stored min is the exact group minimum
    mins = np.moveaxis(m[..., 0], gd, -1).reshape(-1).astype(np.float32)
    assert np.array_equal(mins, xg.min(1))


@pytest.mark.parametrize("bits", [4, 8])
def test_brute_force_nearest_level(bits):
    """Tiny random groups: every code is the nearest integer to (x - min) * scale taken
    in exact rational arithmetic, except within the fp32 rounding band around ties."""
    rng = np.random.default_rng(5)
    B = (1 << bits) - 1
    for trial in range(40):
        x = (rng.standard_normal(32) * rng.choice([0.01, 1.0, 30.0])).astype(np.float16)
        c, m = codec.compress(x, bits, 32, 0)
        q = c.tolist()
        if bits == 4:
            q = []
            for b in c.tolist():
                q += [b & 15, b >> 4]
        mn = Fraction(float(x.min()))
        s = Fraction(float(m[0, 1]))
        r = Fraction(float(x.max())) - mn
        if r == 0:
            assert all(v == 0 for v in q)
            continue
        # the stored scale is the fp16 nearest to B/r (or 65504 when that overflows)
        ideal = Fraction(B) / r
        if ideal <= 65504:
            assert abs(s - ideal) <= ideal * Fraction(1, 2048)
        for xi, qi in zip(x.tolist(), q):
            t = (Fraction(xi) - mn) * s
            assert 0 <= qi <= B
            eta = abs(t) * Fraction(1, 2 ** 22) + Fraction(1, 2 ** 40)
            assert abs(t - qi) <= Fraction(1, 2) + eta
            frac = t - int(t)
            if abs(frac - Fraction(1, 2)) > eta:
                assert qi == min(B, round(t))


def test_layout_invariance_under_transpose():
    """Grouping along a strided dim gives the transposed result of grouping the
    transposed tensor along its contiguous dim (both group the same elements)."""
    x = _sweep_tensor((256, 96), 0, 64, seed=14)
    c0, m0 = codec.compress(x, 4, 64, 0)
    c1, m1 = codec.compress(np.ascontiguousarray(x.T), 4, 64, 1)
    assert np.array_equal(c0, c1.T)
    assert np.array_equal(m0, m1.transpose(1, 0, 2))
    x4 = _sweep_tensor((2, 3, 5, 128), 3, 64, seed=15)
    c3, m3 = codec.compress(x4, 4, 64, 3)
    cT, mT = codec.compress(np.ascontiguousarray(np.moveaxis(x4, 3, 1)), 4, 64, 1)
    assert np.array_equal(c3, np.moveaxis(cT, 1, 3))
    assert np.array_equal(m3, np.moveaxis(mT, 1, 3))


def test_group_locality():
    """Changing one element changes only the codes and metadata of its own group."""
    x = _sweep_tensor((8, 256), 1, 64, seed=16)
    c, m = codec.compress(x, 4, 64, 1)
    x2 = x.copy()
    x2[3, 130] = np.float16(100.0)
    c2, m2 = codec.compress(x2, 4, 64, 1)
    diff_c = np.argwhere(c != c2)
    diff_m = np.argwhere((m != m2).any(-1))
    assert len(diff_m) == 1 and tuple(diff_m[0]) == (3, 2)
    assert np.all(diff_c[:, 0] == 3) and np.all((diff_c[:, 1] // 32) == 2)


def test_saturated_scale():
    """A group whose range is below (2^b-1)/65504 gets the largest fp16 scale."""
    x = np.full(64, 0.1, np.float16)
    x[5] = np.float16(0.1) + np.float16(2.0 ** -14)     # range 2^-14 < 15/65504
    c, m = codec.compress(x, 4, 64, 0)
    assert float(m[0, 1]) == 65504.0                    # 15/2^-14 overflows fp16
    assert int(c[2] >> 4) == 4                          # element 5: 2^-14 * 65504 = 3.998 -> 4
    assert int(c[2] & 15) == 0 and int(c[0]) == 0


@pytest.mark.parametrize("order", [(-0.0, 0.0), (0.0, -0.0)])
@pytest.mark.parametrize("bits", [3, 4, 8])
def test_zero_minimum_is_stored_as_plus_zero(order, bits):
    """A group whose smallest value is a zero (both signs present, in either order, or
    -0 alone) stores min = +0 (bits 0x0000); the codes and the decoded values are those
    of the same group with every -0 replaced by +0."""
    x = np.array([0.5, order[0], 1.0, order[1]] + [0.25] * 28, np.float16)
    c, m = codec.compress(x, bits, 32, 0)
    assert np.ascontiguousarray(m).view(np.uint16)[0, 0] == 0
    xp = np.where(x == 0, np.float16(0.0), x)
    cp, mp = codec.compress(xp, bits, 32, 0)
    assert np.array_equal(c, cp) and np.array_equal(np.ascontiguousarray(m).view(np.uint16),
                                                    np.ascontiguousarray(mp).view(np.uint16))
    y = codec.decompress(c, m, x.shape, bits, 32, 0)
    assert y[1] == 0 and y[3] == 0 and not np.signbit(y[1]) and not np.signbit(y[3])
    xn = np.full(32, -0.0, np.float16)                   # an all -0 group: constant, min +0
    _, mn = codec.compress(xn, bits, 32, 0)
    assert np.ascontiguousarray(mn).view(np.uint16)[0, 0] == 0
