"""Parity of flexq_compress / flexq_decompress (CUDA, through the C ABI) with the
oracle: codes, metadata and decompressed fp16 must agree bit for bit.

Sizes span several tiles with a ragged tail; the sweep sizes (1 MB .. 4 GB of fp16,
[R, 4096], contiguous and strided grouping, 4/8 bits, groups 32/64/128) are checked
on sampled row-blocks, which the oracle computes on its own."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc
from _helpers import assert_bits_equal, to_np, sync_status

pytestmark = pytest.mark.gpu

SMALL = [
    ((37, 4096), 1, 64, 4), ((37, 4096), 1, 32, 4), ((37, 4096), 1, 128, 4), ((37, 4096), 1, 64, 8),
    ((37, 4096), 1, 32, 8), ((37, 4096), 1, 128, 8),
    ((320, 520), 0, 64, 4), ((256, 520), 0, 128, 4), ((96, 520), 0, 32, 8), ((192, 1000), 0, 64, 8),
    ((128, 77), 0, 64, 4), ((64, 5), 0, 32, 8),            # ragged widths: scalar path
    ((3, 5, 7, 128), 3, 64, 4), ((3, 5, 128, 6), 2, 32, 4), ((2, 64, 3, 8), 1, 64, 8),
    ((4096,), 0, 64, 4), ((64,), 0, 64, 4), ((1, 64), 1, 64, 8),
    ((7, 4160), 1, 64, 4), ((9, 2080), 1, 32, 8), ((5, 3200), 1, 128, 4),   # ragged last staged chunk
]


def _run(shape, gd, gs, bits, seed):
    x = synth.codec_tensor(shape, gd, gs, seed)
    cfg = fq.config(bits, gs, gd)
    xd = x.cuda()
    codes, meta = fq.flexq_compress(xd, cfg)
    y = fq.flexq_decompress(codes, meta, shape, cfg)
    sync_status()
    return x.numpy(), codes, meta, y


@pytest.mark.parametrize("shape,gd,gs,bits", SMALL)
def test_codec_bit_exact_small(shape, gd, gs, bits):
    x, codes, meta, y = _run(shape, gd, gs, bits, seed=101)
    rc, rm = oc.compress(x, bits, gs, gd)
    assert_bits_equal(codes, rc, "codes")
    assert_bits_equal(meta, rm, "meta")
    ry = oc.decompress(rc, rm, shape, bits, gs, gd)
    assert_bits_equal(y, ry, "decompressed")


def test_kv_shaped_case_small():
    # [tokens, sequences*heads, head_dim] grouped along head_dim (group_dim 2)
    shape = (17, 6 * 4, 128)
    x, codes, meta, y = _run(shape, 2, 64, 4, seed=102)
    rc, rm = oc.compress(x, 4, 64, 2)
    assert_bits_equal(codes, rc, "codes")
    assert_bits_equal(meta, rm, "meta")


def test_empty_tensor_is_noop():
    cfg = fq.config(4, 64, 1)
    x = torch.empty((0, 4096), dtype=torch.float16, device="cuda")
    codes, meta = fq.flexq_compress(x, cfg)
    y = fq.flexq_decompress(codes, meta, (0, 4096), cfg)
    sync_status()
    assert codes.numel() == 0 and y.numel() == 0


def test_misaligned_pointer_rejected():
    cfg = fq.config(4, 64, 1)
    x = torch.zeros(4 * 4096 + 8, dtype=torch.float16, device="cuda")
    with pytest.raises(fq.FlexError) as e:
        fq.flexq_compress(x[1:1 + 4 * 4096].view(4, 4096), cfg)
    assert e.value.code == fq.FLEX_ERR_ALIGN


def _sample_blocks(R, gs, gd, nsample, rng):
    """Row ranges that are whole groups: rows for gd=1, row-blocks of gs for gd=0."""
    if gd == 1:
        rows = np.unique(np.concatenate([[0, R - 1], rng.integers(0, R, nsample)]))
        return [(int(r), int(r) + 1) for r in rows]
    nb = R // gs
    blocks = np.unique(np.concatenate([[0, nb - 1], rng.integers(0, nb, nsample)]))
    return [(int(b) * gs, int(b) * gs + gs) for b in blocks]


SWEEP = [(mb, gd, gs, bits) for mb in (1, 16, 256, 1024, 4096) for gd, gs, bits in
         ((1, 64, 4), (0, 64, 4))] + [(256, 1, 32, 4), (256, 1, 128, 4), (256, 1, 64, 8),
                                       (256, 0, 128, 8), (256, 0, 32, 4)]


@pytest.mark.parametrize("mb,gd,gs,bits", SWEEP)
def test_codec_sweep_sampled(mb, gd, gs, bits):
    """Full sweep sizes, in the launch configuration the benchmark times; the oracle
    checks sampled whole groups, the GPU's own round trip checks everything else
    (decompress of compress must stay within the quantiser's error bound)."""
    R = synth.codec_rows_for_bytes(mb << 20)
    R -= R % 128
    shape = (R, 4096)
    x = synth.codec_tensor(shape, gd, gs, seed=200 + mb, device="cuda")
    cfg = fq.config(bits, gs, gd)
    codes, meta = fq.flexq_compress(x, cfg)
    y = fq.flexq_decompress(codes, meta, shape, cfg)
    sync_status()
    rng = np.random.default_rng(mb)
    for (r0, r1) in _sample_blocks(R, gs, gd, 6, rng):
        xs = to_np(x[r0:r1])
        rc, rm = oc.compress(xs, bits, gs, gd)
        if gd == 0:
            c_rows = slice(r0 * bits // 8, r1 * bits // 8)
            m_rows = slice(r0 // gs, r1 // gs)
        else:
            c_rows = slice(r0, r1)
            m_rows = slice(r0, r1)
        assert_bits_equal(codes[c_rows], rc, f"codes rows {r0}:{r1}")
        assert_bits_equal(meta[m_rows], rm, f"meta rows {r0}:{r1}")
        assert_bits_equal(y[r0:r1], oc.decompress(rc, rm, xs.shape, bits, gs, gd), f"y rows {r0}:{r1}")
    # everywhere: |y - x| within range/(2(2^b-1)) (+ fp16 rounding), via the GPU's meta
    B = (1 << bits) - 1
    xf = x.float()
    yf = y.float()
    if gd == 0:
        xg = xf.view(R // gs, gs, 4096).transpose(1, 2).reshape(-1, gs)
        yg = yf.view(R // gs, gs, 4096).transpose(1, 2).reshape(-1, gs)
    else:
        xg = xf.view(-1, gs)
        yg = yf.view(-1, gs)
    r = (xg.max(1).values - xg.min(1).values)
    quant = torch.clamp(r / (2 * B) * (1 + 2 ** -10), min=0.5 / 65504 * (1 + 2 ** -10))
    quant = torch.where(r == 0, torch.zeros_like(r), quant)
    bound = quant[:, None] + 2 ** -11 * yg.abs() + 2 ** -22 * (xg.min(1).values.abs() + r)[:, None] + 2 ** -25
    assert bool(((yg - xg).abs() <= bound).all())
    del x, codes, meta, y, xf, yf, xg, yg
    torch.cuda.empty_cache()
