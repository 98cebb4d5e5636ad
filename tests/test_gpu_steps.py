"""Parity of the single hot-path steps (LayerNorm, store_cache) with the oracle."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc
from oracle import layer as ol
from _helpers import assert_bits_equal, to_np, sync_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("h,rows", [(768, 5), (2048, 33), (7168, 3), (12288, 2), (64, 7)])
def test_layernorm(h, rows):
    x = synth.activations((rows, h), 31)
    p = synth.layer_params(h, 8, 31)
    g, b = p["ln1_g"], p["ln1_b"]
    y = torch.empty((rows, h), dtype=torch.float16, device="cuda")
    fq.flex_layernorm(x.cuda(), g.cuda(), b.cuda(), y, rows, h)
    sync_status()
    ref = ol.layer_norm(x.numpy(), g.numpy(), b.numpy())
    err = np.abs(to_np(y).astype(np.float64) - ref)
    # fp32 statistics, one fp16 rounding of the output
    assert np.all(err <= 2.0 ** -10 * np.abs(ref) + 2e-3), float(err.max())


@pytest.mark.parametrize("batch,nh,d,bits,gs,pos", [(4, 12, 64, 4, 64, 0), (3, 5, 128, 4, 64, 17),
                                                    (2, 3, 128, 8, 64, 5), (5, 2, 64, 4, 32, 9)])
def test_append_kv_bit_exact(batch, nh, d, bits, gs, pos):
    h = nh * d
    qkv = synth.activations((batch, 3 * h), 32)        # rows [q | k | v]
    cache = fq.FlexKVCache(batch + 1, nh, d, 24, bits, gs)
    q = qkv.cuda()
    fq.flex_append_kv(cache, q[:, h:], q[:, 2 * h:], 3 * h, batch, pos)
    sync_status()
    for which, codes, meta in ((1, cache.k_codes, cache.k_meta), (2, cache.v_codes, cache.v_meta)):
        src = qkv.numpy()[:, which * h:(which + 1) * h].reshape(batch, nh, d)
        rc, rm = oc.compress(np.ascontiguousarray(src), bits, gs, 2)
        assert_bits_equal(codes[:batch, :, pos], rc, "codes")
        assert_bits_equal(meta[:batch, :, pos], rm, "meta")
        # nothing else was written
        mask = torch.ones_like(codes, dtype=torch.bool)
        mask[:batch, :, pos] = False
        assert int(codes[mask].count_nonzero()) == 0
