"""Group-wise asymmetric min/max quantiser (oracle; test infrastructure only).

Statement followed: the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 6.3 - ``compress`` splits a
tensor along ``group_dim`` into groups of ``group_size`` elements, keeps per group a
fp16 scale, and stores ``num_bits``-bit unsigned codes, two 4-bit codes per uint8,
in a data tensor of shape
``shape[:group_dim] + (num_groups * group_size * num_bits // 8,) + shape[group_dim+1:]``.
The quantisation formula is the min/max one of the method:
``q = clamp(round((x - min) * (2^b - 1) / (max - min)), 0, 2^b - 1)`` and
``x^ = q * (max - min) / (2^b - 1) + min``.

Readings where the pages leave a step open (each listed in the design notes):

* metadata per group is the pair ``{min, scale}`` in fp16 (stored as one half2),
  ``scale = (2^b - 1) / (max - min)``;
* codes are computed with the *stored* fp16 scale, so codes and metadata agree;
* rounding is round-half-to-even;
* ``max == min``: scale 0, all codes 0, decompression returns min exactly;
* a scale above the fp16 range saturates to 65504 (codes stay <= 2^b - 1);
* 4-bit packing puts the even element of a pair in the low nibble;
* decompression multiplies by the reciprocal of the scale, rounded once per group:
  ``x^ = q * (1/scale) + min`` as two separately rounded fp32 operations, then one
  rounding to fp16.

Variants (readings of what the pages only name: the ``symmetric`` flag of the
configuration, "int3/int4" group-wise quantisation, and ``num_groups`` groups along
group_dim):

* ``symmetric=True`` (absmax): ``B = 2^(b-1) - 1``, ``scale = fp16(B / max|x|)`` (0 for an
  all-zero group, 65504 on overflow), signed codes ``q = clamp(rint(x * scale), -B, B)``
  stored offset-binary as ``q + B`` in b bits, metadata ``{0, scale}``, and
  ``x^ = fp16(fl((u - B) * fl(1/scale)))`` (0 when scale is 0);
* ``num_bits=3``: levels 0..7; the codes of a group form a little-endian bit stream,
  code j in bits [3j, 3j+3), i.e. 8 codes in every 3 bytes;
* a group dimension that is not a multiple of group_size is zero-padded to whole
  groups before quantisation (num_groups = ceil(dim / group_size) groups along it, as in
  the pages' packed shape), and decompression returns the original extent.

All arithmetic is IEEE binary32 with every operation rounded on its own: numpy
float32 ufuncs perform no contraction, and float32 -> float16 casts round to
nearest-even.
"""
from __future__ import annotations

import numpy as np

SUPPORTED_BITS = (3, 4, 8)
SUPPORTED_GROUPS = (32, 64, 128)
FP16_MAX = np.float16(65504.0)


def _check(shape, num_bits, group_size, group_dim, symmetric):
    if num_bits not in SUPPORTED_BITS:
        raise ValueError(f"num_bits {num_bits} not in {SUPPORTED_BITS}")
    if group_size not in SUPPORTED_GROUPS:
        raise ValueError(f"group_size {group_size} not in {SUPPORTED_GROUPS}")
    nd = len(shape)
    if not 1 <= nd <= 4:
        raise ValueError("rank must be 1..4")
    return group_dim % nd


def num_groups(shape, group_size=64, group_dim=0):
    """Groups along group_dim: ceil(dim / group_size) (a partial last group is zero-padded)."""
    shape = tuple(int(d) for d in shape)
    gd = group_dim % len(shape)
    return -(-shape[gd] // group_size)


def codes_shape(shape, num_bits=4, group_size=64, group_dim=0):
    """Packed data shape of the pages: shape[:gd] + (ng*gs*bits/8,) + shape[gd+1:]."""
    shape = tuple(int(d) for d in shape)
    gd = group_dim % len(shape)
    ng = num_groups(shape, group_size, group_dim)
    return shape[:gd] + (ng * group_size * num_bits // 8,) + shape[gd + 1:]


def meta_shape(shape, num_bits=4, group_size=64, group_dim=0):
    """Metadata shape: one {min, scale} fp16 pair per group -> shape[:gd]+(ng,)+shape[gd+1:]+(2,)."""
    shape = tuple(int(d) for d in shape)
    gd = group_dim % len(shape)
    ng = num_groups(shape, group_size, group_dim)
    return shape[:gd] + (ng,) + shape[gd + 1:] + (2,)


def _groups(x, gd, group_size):
    """View with the group dimension moved last, zero-padded to whole groups and split
    into (num_groups, group_size)."""
    xm = np.moveaxis(x, gd, -1)
    lead = xm.shape[:-1]
    ng = -(-xm.shape[-1] // group_size)
    pad = ng * group_size - xm.shape[-1]
    if pad:
        xm = np.concatenate([xm, np.zeros(lead + (pad,), xm.dtype)], axis=-1)
    return xm.reshape(lead + (ng, group_size))


def group_params(g32, num_bits):
    """Per group: min, fp16 scale. g32: float32 array [..., group_size]."""
    levels = np.float32((1 << num_bits) - 1)
    mn = g32.min(axis=-1) + np.float32(0)                  # a zero minimum is +0 (reading R26)
    mx = g32.max(axis=-1)
    r = mx - mn                                            # fp32, rounded once
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        s32 = np.where(r > 0, levels / np.where(r > 0, r, np.float32(1)), np.float32(0))
        s32 = s32.astype(np.float32)
        s16 = s32.astype(np.float16)                       # round to nearest even
    s16 = np.where(np.isinf(s16), FP16_MAX, s16).astype(np.float16)
    return mn.astype(np.float32), s16


def quantize_groups(g32, mn, s16, num_bits):
    """Codes of every element: clamp(rint((x - min) * scale), 0, 2^b - 1)."""
    levels = np.float32((1 << num_bits) - 1)
    s = s16.astype(np.float32)[..., None]
    d = (g32 - mn[..., None]).astype(np.float32)           # one rounding
    t = (d * s).astype(np.float32)                         # one rounding
    q = np.clip(np.rint(t), np.float32(0), levels)
    return q.astype(np.uint8)


def symmetric_params(g32, num_bits):
    """Per group (absmax form): fp16 scale = (2^(b-1) - 1) / max|x|, 0 for a zero group."""
    levels = np.float32((1 << (num_bits - 1)) - 1)
    a = np.abs(g32).max(axis=-1)                           # exact
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        s32 = np.where(a > 0, levels / np.where(a > 0, a, np.float32(1)), np.float32(0)).astype(np.float32)
        s16 = s32.astype(np.float16)
    return np.where(np.isinf(s16), FP16_MAX, s16).astype(np.float16)


def quantize_symmetric(g32, s16, num_bits):
    """Offset-binary codes q + B of q = clamp(rint(x * scale), -B, B)."""
    B = np.float32((1 << (num_bits - 1)) - 1)
    t = (g32 * s16.astype(np.float32)[..., None]).astype(np.float32)    # one rounding
    q = np.clip(np.rint(t), -B, B)
    return (q + B).astype(np.uint8)


def pack(q, num_bits):
    """Pack codes along the last axis: 4-bit -> byte j = q[2j] | q[2j+1] << 4; 3-bit ->
    a little-endian bit stream (code j in bits [3j, 3j+3)); 8-bit -> one per byte."""
    if num_bits == 8:
        return q.astype(np.uint8)
    if num_bits == 3:
        n = q.shape[-1]
        bits = ((q[..., :, None].astype(np.uint16) >> np.arange(3, dtype=np.uint16)) & 1).astype(np.uint8)
        bits = bits.reshape(q.shape[:-1] + (3 * n,))                      # bit 3j + i = bit i of q[j]
        return np.packbits(bits, axis=-1, bitorder="little")
    lo = q[..., 0::2].astype(np.uint8)
    hi = q[..., 1::2].astype(np.uint8)
    return (lo | (hi << 4)).astype(np.uint8)


def unpack(b, num_bits):
    """Inverse of pack along the last axis."""
    if num_bits == 8:
        return b.astype(np.uint8)
    if num_bits == 3:
        bits = np.unpackbits(b, axis=-1, bitorder="little")             # 8 bits per byte
        n = bits.shape[-1] // 3
        bits = bits.reshape(b.shape[:-1] + (n, 3)).astype(np.uint8)
        return (bits[..., 0] | (bits[..., 1] << 1) | (bits[..., 2] << 2)).astype(np.uint8)
    out = np.empty(b.shape[:-1] + (b.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = b & 0x0F
    out[..., 1::2] = b >> 4
    return out


def compress(x16, num_bits=4, group_size=64, group_dim=0, symmetric=False):
    """Compress a fp16 tensor. Returns (codes uint8, meta float16[..., 2] = {min, scale}).

    codes has the pages' packed data shape; meta has shape
    shape[:gd] + (num_groups,) + shape[gd+1:] + (2,) ({0, scale} in the symmetric form).
    """
    x = np.asarray(x16)
    if x.dtype != np.float16:
        raise TypeError("input must be float16")
    gd = _check(x.shape, num_bits, group_size, group_dim, symmetric)
    g = _groups(x, gd, group_size).astype(np.float32)      # exact widening (pad: zeros)
    if symmetric:
        s16 = symmetric_params(g, num_bits)
        q = quantize_symmetric(g, s16, num_bits)
        mn16 = np.zeros(s16.shape, np.float16)
    else:
        mn, s16 = group_params(g, num_bits)
        q = quantize_groups(g, mn, s16, num_bits)
        mn16 = mn.astype(np.float16)
    packed = pack(q, num_bits)                              # [..., ng, gs*bits/8]
    lead = packed.shape[:-2]
    packed = packed.reshape(lead + (packed.shape[-2] * packed.shape[-1],))
    codes = np.ascontiguousarray(np.moveaxis(packed, -1, gd))
    meta = np.stack([mn16, s16], axis=-1)                   # [..., ng, 2]
    meta = np.ascontiguousarray(np.moveaxis(meta, -2, gd))
    return codes, meta


def decompress(codes, meta, shape, num_bits=4, group_size=64, group_dim=0, symmetric=False):
    """Rebuild the fp16 tensor: x^ = q * (1/scale) + min (scale 0 -> min); symmetric:
    x^ = (u - B) * (1/scale) (scale 0 -> 0)."""
    shape = tuple(int(d) for d in shape)
    gd = _check(shape, num_bits, group_size, group_dim, symmetric)
    cm = np.moveaxis(np.asarray(codes, dtype=np.uint8), gd, -1)
    lead = cm.shape[:-1]
    ng = num_groups(shape, group_size, group_dim)
    per = group_size * num_bits // 8
    q = unpack(cm.reshape(lead + (ng, per)), num_bits).astype(np.float32)
    mm = np.moveaxis(np.asarray(meta, dtype=np.float16), gd, -2)  # [..., ng, 2]
    mn = mm[..., 0].astype(np.float32)
    s = mm[..., 1].astype(np.float32)
    with np.errstate(divide="ignore"):
        step = np.where(s > 0, np.float32(1) / np.where(s > 0, s, np.float32(1)), np.float32(0))
    step = step.astype(np.float32)
    if symmetric:
        B = np.float32((1 << (num_bits - 1)) - 1)
        qs = (q - B).astype(np.float32)                     # exact (small integers)
        xh = (qs * step[..., None]).astype(np.float32)      # one rounding; scale 0 -> step 0 -> 0
    else:
        prod = (q * step[..., None]).astype(np.float32)     # one rounding
        xh = (prod + mn[..., None]).astype(np.float32)      # one rounding
        xh = np.where((s > 0)[..., None], xh, mn[..., None])
    y = xh.astype(np.float16).reshape(lead + (ng * group_size,))[..., :shape[gd]]
    return np.ascontiguousarray(np.moveaxis(y, -1, gd))


def compressed_bytes(shape, num_bits=4, group_size=64, group_dim=0):
    """Bytes of codes + metadata (fp16 min and fp16 scale per group)."""
    return int(np.prod(codes_shape(shape, num_bits, group_size, group_dim))) + \
        int(np.prod(meta_shape(shape, num_bits, group_size, group_dim))) * 2
