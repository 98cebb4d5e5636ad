"""flexq_compress / flexq_decompress for the codec variants - 3-bit codes, the symmetric
(absmax) form and zero-padded partial groups - bit-exact against the oracle codec on
contiguous, strided and KV-shaped tensors, small and at 256 MB (sampled). Contiguous
groups whose extent is a multiple of 8 (the last three small shapes, partial last groups
included, and the 256 MB contiguous cases) take the vectorised variant kernels; the
other shapes take the one-thread-per-group kernels."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc
from _helpers import assert_bits_equal, to_np, sync_status

pytestmark = pytest.mark.gpu


def _run(x, bits, gs, gd, sym):
    cfg = fq.config(bits, gs, gd, int(sym))
    codes, meta = fq.flexq_compress(x.cuda(), cfg)
    y = fq.flexq_decompress(codes, meta, x.shape, cfg)
    sync_status()
    return codes, meta, y


@pytest.mark.parametrize("shape,gd", [((16, 256), 1), ((256, 24), 0), ((3, 100), 1), ((70, 5), 0),
                                      ((2, 5, 96, 3), 2), ((4, 3, 130), -1),
                                      ((5, 200), 1), ((6, 1000), -1), ((3, 7, 136), 2)])
@pytest.mark.parametrize("bits,sym", [(3, False), (3, True), (4, True), (8, True), (4, False), (8, False)])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_variants_bit_exact(shape, gd, bits, sym, gs):
    x = synth.codec_tensor(tuple(d if i != gd % len(shape) else -(-d // gs) * gs for i, d in enumerate(shape)),
                           gd, gs, seed=bits * 100 + gs)
    x = x[tuple(slice(0, d) for d in shape)].contiguous()              # a partial last group
    x.view(-1)[:5] = torch.tensor([3e-5, 3.01e-5, 0.0, -0.0, 2.0], dtype=torch.float16)
    codes, meta, y = _run(x, bits, gs, gd, sym)
    rc, rm = oc.compress(x.numpy(), bits, gs, gd, symmetric=sym)
    assert_bits_equal(codes, rc, "codes")
    assert_bits_equal(meta, rm, "meta")
    assert_bits_equal(y, oc.decompress(rc, rm, x.shape, bits, gs, gd, symmetric=sym), "decompressed")


@pytest.mark.parametrize("bits,sym,gd", [(3, False, 1), (4, True, 1), (3, True, 0), (8, True, 1), (3, True, 1)])
def test_variants_256mb_sampled(bits, sym, gd):
    """256 MB fp16 [32768, 4096]: sampled groups equal the oracle's."""
    shape = (32768, 4096)
    x = synth.codec_tensor(shape, gd, 64, seed=11, device="cuda")
    cfg = fq.config(bits, 64, gd, int(sym))
    codes, meta = fq.flexq_compress(x, cfg)
    y = fq.flexq_decompress(codes, meta, shape, cfg)
    sync_status()
    if gd == 1:
        rows = [0, 1, 12345, 32767]
        xs = to_np(x[rows])
        rc, rm = oc.compress(xs, bits, 64, 1, symmetric=sym)
        assert_bits_equal(codes[rows], rc, "codes")
        assert_bits_equal(meta[rows], rm, "meta")
        assert_bits_equal(y[rows], oc.decompress(rc, rm, xs.shape, bits, 64, 1, symmetric=sym), "y")
    else:
        cols = [0, 7, 4095]
        for g in (0, 200, 511):                         # groups of 64 rows along dim 0
            xs = to_np(x[g * 64:(g + 1) * 64][:, cols])
            rc, rm = oc.compress(xs, bits, 64, 0, symmetric=sym)
            cb = 64 * bits // 8
            assert_bits_equal(codes[g * cb:(g + 1) * cb][:, cols], rc, "codes")
            assert_bits_equal(meta[g:g + 1][:, cols], rm, "meta")
            assert_bits_equal(y[g * 64:(g + 1) * 64][:, cols], oc.decompress(rc, rm, xs.shape, bits, 64, 0,
                                                                            symmetric=sym), "y")


@pytest.mark.parametrize("bits,sym,gs", [(4, False, 64), (8, False, 64), (3, True, 128)])
def test_variants_partial_groups_large_sampled(bits, sym, gs):
    """[65536, 1000] (131 MB fp16): every row ends in a partial group, and each thread of
    the variant kernels walks about ten groups across row boundaries (grid stride), so
    the row and in-row index it steps forward are checked; 66 sampled rows equal the
    oracle's."""
    shape = (65536, 1000)
    full = (shape[0], -(-shape[1] // gs) * gs)
    x = synth.codec_tensor(full, 1, gs, seed=12, device="cuda")[:, :shape[1]].contiguous()
    cfg = fq.config(bits, gs, 1, int(sym))
    codes, meta = fq.flexq_compress(x, cfg)
    y = fq.flexq_decompress(codes, meta, shape, cfg)
    sync_status()
    rng = np.random.default_rng(5)
    rows = sorted({0, 1, shape[0] - 1, *rng.integers(0, shape[0], 63).tolist()})
    xs = to_np(x[rows])
    rc, rm = oc.compress(xs, bits, gs, 1, symmetric=sym)
    assert_bits_equal(codes[rows], rc, "codes")
    assert_bits_equal(meta[rows], rm, "meta")
    assert_bits_equal(y[rows], oc.decompress(rc, rm, xs.shape, bits, gs, 1, symmetric=sym), "y")
