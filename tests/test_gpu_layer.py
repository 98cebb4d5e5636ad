"""End-to-end parity of flex_prefill_layer / flex_decode_layer (C ABI) with the
oracle layer: prefill of the prompt, then decode steps, each side keeping its own
int4 KV cache. Layer outputs: max|err| <= 1e-2 max|ref| + 1e-3 at every step."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc
from oracle import layer as ol
from _helpers import assert_layer_close, assert_bits_equal, to_np, sync_status

pytestmark = pytest.mark.gpu


def _setup(cfg, seed, device="cpu"):
    raw = synth.layer_params(cfg["h"], cfg["ffn"], seed, device=device)
    return raw


def _ws(layer, batch, seq):
    return torch.zeros(fq.flex_workspace_bytes(layer, batch, seq), dtype=torch.uint8, device="cuda")


def _qkv_offset(batch, seq, h):
    T = batch * seq
    return (T * h * 2 + 255) // 256 * 256


@pytest.mark.parametrize("bits", [4, 8])
def test_opt125m_prefill_and_decode_full(bits):
    cfg = dict(synth.WORKLOADS["opt-125m"])
    b, s, h, nh, d = cfg["batch"], cfg["prompt"], cfg["h"], cfg["n_heads"], cfg["head_dim"]
    steps = cfg["decode_steps"]
    max_seq = s + steps
    raw = _setup(cfg, cfg["seed"])
    layer = fq.FlexLayer(raw, nh)
    cache = fq.FlexKVCache(b, nh, d, max_seq, bits, 64)
    PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
    W = ol.dequant_all(PQ)
    ocache = ol.KVCache(b, nh, max_seq, d, bits, 64)

    x = synth.activations((b, s, h), cfg["seed"])
    y = torch.empty((b, s, h), dtype=torch.float16, device="cuda")
    ws = _ws(layer, b, s)
    fq.flex_prefill_layer(layer, cache, x.cuda(), y, b, s, ws)
    sync_status()
    ref = ol.prefill_layer(x.numpy(), PQ, ocache, nh, W=W)
    assert_layer_close(y, ref, "prefill")

    # cache slots [0, s): exactly the quantiser applied to the layer's own fp16 k/v
    qkv = ws[_qkv_offset(b, s, h):].view(torch.float16)[: b * s * 3 * h].view(b, s, 3 * h)
    k16 = qkv[..., h:2 * h].reshape(b, s, nh, d).permute(0, 2, 1, 3).contiguous()
    kc, km = fq.flexq_compress(k16, fq.config(bits, 64, 3))
    sync_status()
    assert torch.equal(cache.k_codes[:, :, :s], kc) and torch.equal(cache.k_meta[:, :, :s], km)
    # ... and that k/v agree with the oracle's within the quantiser's bound (+ fp16 slack)
    kd = fq.flexq_decompress(cache.k_codes[:, :, :s].contiguous(), cache.k_meta[:, :, :s].contiguous(),
                             (b, nh, s, d), fq.config(bits, 64, 3)).float()
    kref = ol.KVCache.load(ocache, s)[0]
    r = np.abs(kref).max()
    assert float(np.abs(to_np(kd) - kref).max()) <= 2 * r / ((1 << bits) - 1) + 2e-2

    wsd = _ws(layer, b, 1)
    for t in range(steps):
        xd = synth.decode_inputs(b, h, t, cfg["seed"])
        yd = torch.empty((b, h), dtype=torch.float16, device="cuda")
        fq.flex_decode_layer(layer, cache, xd.cuda(), yd, b, s + t, wsd)
        sync_status()
        refd = ol.decode_layer(xd.numpy(), PQ, ocache, s + t, nh, W=W)
        assert_layer_close(yd, refd, f"decode step {t}")


def test_decode_degenerate_pos0_and_batch_subset():
    """pos 0 (no cached keys: the token attends to itself) and a decode batch smaller
    than the cache's."""
    cfg = dict(synth.WORKLOADS["opt-125m"])
    h, nh, d = cfg["h"], cfg["n_heads"], cfg["head_dim"]
    raw = _setup(cfg, 9)
    layer = fq.FlexLayer(raw, nh)
    cache = fq.FlexKVCache(5, nh, d, 4)
    PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
    W = ol.dequant_all(PQ)
    ocache = ol.KVCache(3, nh, 4, d)
    xd = synth.decode_inputs(3, h, 0, 9)
    yd = torch.empty((3, h), dtype=torch.float16, device="cuda")
    fq.flex_decode_layer(layer, cache, xd.cuda(), yd, 3, 0, _ws(layer, 3, 1))
    sync_status()
    assert_layer_close(yd, ol.decode_layer(xd.numpy(), PQ, ocache, 0, nh, W=W), "pos 0")
    assert int(cache.k_codes[3:].count_nonzero()) == 0


def test_opt13b_sampled_sequences():
    """opt-1.3b shape at full size (32 sequences, prompt 512, then decode steps); the
    oracle follows two sampled sequences (sequences are independent)."""
    cfg = dict(synth.WORKLOADS["opt-1.3b"])
    b, s, h, nh, d = cfg["batch"], cfg["prompt"], cfg["h"], cfg["n_heads"], cfg["head_dim"]
    steps = 3
    max_seq = s + cfg["decode_steps"]
    raw = _setup(cfg, cfg["seed"])
    layer = fq.FlexLayer(raw, nh)
    cache = fq.FlexKVCache(b, nh, d, max_seq)
    rows = [0, b - 1]
    PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
    W = ol.dequant_all(PQ)
    ocache = ol.KVCache(len(rows), nh, max_seq, d)
    x = synth.activations((b, s, h), cfg["seed"])
    y = torch.empty((b, s, h), dtype=torch.float16, device="cuda")
    fq.flex_prefill_layer(layer, cache, x.cuda(), y, b, s, _ws(layer, b, s))
    sync_status()
    ref = ol.prefill_layer(x.numpy()[rows], PQ, ocache, nh, W=W)
    assert_layer_close(y[rows], ref, "prefill (sampled)")
    wsd = _ws(layer, b, 1)
    for t in range(steps):
        xd = synth.decode_inputs(b, h, t, cfg["seed"])
        yd = torch.empty((b, h), dtype=torch.float16, device="cuda")
        fq.flex_decode_layer(layer, cache, xd.cuda(), yd, b, s + t, wsd)
        sync_status()
        refd = ol.decode_layer(xd.numpy()[rows], PQ, ocache, s + t, nh, W=W)
        assert_layer_close(yd[rows], refd, f"decode step {t} (sampled)")


def test_layer_bad_args():
    cfg = dict(synth.WORKLOADS["opt-125m"])
    raw = _setup(cfg, 1)
    layer = fq.FlexLayer(raw, cfg["n_heads"])
    cache = fq.FlexKVCache(2, cfg["n_heads"], cfg["head_dim"], 8)
    x = torch.zeros((2, cfg["h"]), dtype=torch.float16, device="cuda")
    y = torch.zeros_like(x)
    ws = _ws(layer, 2, 1)
    with pytest.raises(fq.FlexError) as e:
        fq.flex_decode_layer(layer, cache, x, y, 2, 8, ws)
    assert e.value.code == fq.FLEX_ERR_SHAPE
    with pytest.raises(fq.FlexError) as e:
        fq.flex_decode_layer(layer, cache, x, y, 2, 0, ws[:16])
    assert e.value.code == fq.FLEX_ERR_WORKSPACE
    with pytest.raises(fq.FlexError) as e:
        fq.flex_decode_layer(layer, cache, x, x, 2, 0, ws)
    assert e.value.code == fq.FLEX_ERR_INVALID_ARG
