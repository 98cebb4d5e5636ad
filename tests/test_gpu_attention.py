"""Parity of decode attention (int4/int8 cache, split-KV) and prefill attention
(causal, fresh fp16 q/k/v) with the oracle."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import layer as ol
from _helpers import assert_layer_close, to_np, sync_status

pytestmark = pytest.mark.gpu


def _decode_case(batch, nh, d, bits, gs, pos, seed, max_seq=None):
    max_seq = max_seq or pos + 3
    h = nh * d
    kh, vh = synth.kv_history(batch, nh, max(pos, 1), d, seed)
    cache = fq.FlexKVCache(batch, nh, d, max_seq, bits, gs)
    oc = ol.KVCache(batch, nh, max_seq, d, bits, gs)
    if pos > 0:
        cache.fill_from(kh[:, :, :pos].cuda(), vh[:, :, :pos].cuda())
        oc.store(kh[:, :, :pos].numpy(), vh[:, :, :pos].numpy(), 0)
    qkv = synth.activations((batch, 3 * h), seed + 1)
    qkv[:, :h] *= 0.125
    g = qkv.cuda()
    o = torch.empty((batch, h), dtype=torch.float16, device="cuda")
    ws = torch.empty(max(16, fq.flex_decode_attention_ws_bytes(cache, batch, pos)), dtype=torch.uint8, device="cuda")
    fq.flex_decode_attention(cache, g[:, :h], g[:, h:], g[:, 2 * h:], 3 * h, o, batch, pos, ws)
    sync_status()
    q = qkv.numpy()
    ref = ol.decode_attention(q[:, :h].reshape(batch, nh, d), q[:, h:2 * h].reshape(batch, nh, d),
                              q[:, 2 * h:].reshape(batch, nh, d), oc, pos)
    return o, ref.reshape(batch, h)


@pytest.mark.parametrize("batch,nh,d,bits,gs,pos", [
    (4, 12, 64, 4, 64, 0), (4, 12, 64, 4, 64, 1), (4, 12, 64, 4, 64, 37), (4, 12, 64, 4, 64, 135),
    (3, 5, 128, 4, 64, 130), (2, 4, 128, 8, 64, 77), (2, 3, 64, 4, 32, 200), (1, 2, 128, 4, 32, 543),
    (32, 32, 64, 4, 64, 543), (2, 2, 64, 8, 32, 9000)])
def test_decode_attention(batch, nh, d, bits, gs, pos):
    o, ref = _decode_case(batch, nh, d, bits, gs, pos, seed=pos + d)
    assert_layer_close(o, ref, f"decode attn pos={pos}")


def test_decode_attention_full_size_sampled():
    """opt-175b shape (144 sequences, 96 heads x 128, pos 543): sampled sequences."""
    batch, nh, d, pos = 144, 96, 128, 543
    h = nh * d
    max_seq = 544
    kh, vh = synth.kv_history(batch, nh, pos, d, 77, device="cuda")
    cache = fq.FlexKVCache(batch, nh, d, max_seq)
    cache.fill_from(kh, vh)
    qkv = synth.activations((batch, 3 * h), 78, device="cuda")
    qkv[:, :h] *= 0.088
    o = torch.empty((batch, h), dtype=torch.float16, device="cuda")
    ws = torch.empty(fq.flex_decode_attention_ws_bytes(cache, batch, pos), dtype=torch.uint8, device="cuda")
    fq.flex_decode_attention(cache, qkv[:, :h], qkv[:, h:], qkv[:, 2 * h:], 3 * h, o, batch, pos, ws)
    sync_status()
    rows = [0, 71, 143]
    oc = ol.KVCache(len(rows), nh, max_seq, d)
    oc.store(to_np(kh[rows]), to_np(vh[rows]), 0)
    q = to_np(qkv[rows])
    ref = ol.decode_attention(q[:, :h].reshape(-1, nh, d), q[:, h:2 * h].reshape(-1, nh, d),
                              q[:, 2 * h:].reshape(-1, nh, d), oc, pos)
    assert_layer_close(o[rows], ref.reshape(len(rows), h), "opt-175b decode attention")


@pytest.mark.parametrize("batch,seq,nh,d", [(2, 1, 2, 64), (2, 77, 3, 64), (1, 200, 2, 128), (3, 64, 4, 128),
                                            (1, 513, 1, 64), (4, 128, 12, 64)])
def test_prefill_attention(batch, seq, nh, d):
    h = nh * d
    qkv = synth.activations((batch, seq, 3 * h), seq + d)
    qkv[..., :h] *= d ** -0.5
    g = qkv.cuda()
    o = torch.empty((batch, seq, h), dtype=torch.float16, device="cuda")
    fq.flex_prefill_attention(g[..., :h], g[..., h:], g[..., 2 * h:], 3 * h, o, batch, seq, nh, d)
    sync_status()
    q = qkv.numpy()
    ref = ol.prefill_attention(q[..., :h].reshape(batch, seq, nh, d), q[..., h:2 * h].reshape(batch, seq, nh, d),
                               q[..., 2 * h:].reshape(batch, seq, nh, d))
    assert_layer_close(o, ref.reshape(batch, seq, h), f"prefill attn s={seq}")


@pytest.mark.parametrize("batch,nh,d,gs,pos,padded", [
    (20, 40, 128, 64, 300, True),      # 800 pairs: beyond one wave of 4 CTAs x 148 SMs
    (20, 40, 128, 32, 257, False),     # a one-key last stage
    (40, 32, 64, 64, 200, True),       # 1280 pairs: beyond one wave of 7 CTAs x 148 SMs
    (40, 32, 64, 32, 128, False),      # exactly one stage per pair
])
def test_decode_attention_many_pairs_every_row(batch, nh, d, gs, pos, padded):
    """Single-split decode with more (sequence, head) pairs than one wave of CTAs: each
    CTA walks several pairs with one copy ring running across them. Every row is
    compared (not a sample), so a pair that picks up its neighbour's keys, query or
    fresh key/value, or a stale softmax state, fails."""
    h = nh * d
    vf = [(37 * b) % (pos + 1) if padded else 0 for b in range(batch)]
    if padded:
        vf[1] = pos                    # only the new token is visible
    vft = torch.tensor(vf, dtype=torch.int32, device="cuda") if padded else None
    kh, vh = synth.kv_history(batch, nh, pos, d, pos + d + gs)
    cache = fq.FlexKVCache(batch, nh, d, pos + 1, 4, gs, valid_from=vft)
    cache.fill_from(kh.cuda(), vh.cuda())
    oc = ol.KVCache(batch, nh, pos + 1, d, 4, gs)
    oc.store(kh.numpy(), vh.numpy(), 0)
    qkv = synth.activations((batch, 3 * h), pos + 5)
    qkv[:, :h] *= d ** -0.5
    g = qkv.cuda()
    o = torch.full((batch, h), float("nan"), dtype=torch.float16, device="cuda")
    ws = torch.empty(max(16, fq.flex_decode_attention_ws_bytes(cache, batch, pos)), dtype=torch.uint8, device="cuda")
    fq.flex_decode_attention(cache, g[:, :h], g[:, h:2 * h], g[:, 2 * h:], 3 * h, o, batch, pos, ws)
    sync_status()
    q = qkv.numpy()
    ref = ol.decode_attention(q[:, :h].reshape(-1, nh, d), q[:, h:2 * h].reshape(-1, nh, d),
                              q[:, 2 * h:].reshape(-1, nh, d), oc, pos, valid_from=vf if padded else None)
    assert_layer_close(o, ref.reshape(batch, h), f"decode attention, {batch * nh} pairs, pos={pos}")
