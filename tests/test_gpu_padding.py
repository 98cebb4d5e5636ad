"""Left padding (variable prompt lengths) on the GPU: flex_kv_cache.valid_from and the
valid_from argument of flex_prefill_attention, against the oracle's masked attention
and layer (prompts padded on the left; no query attends to a pad key; a pad query gets
a zero attention output). Tolerance: max|err| <= 1e-2 max|ref| + 1e-3."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import layer as ol
from _helpers import assert_layer_close, to_np, sync_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("batch,nh,d,bits,pos,vf", [
    (3, 4, 64, 4, 300, [0, 17, 299]),          # one split per pair at this size
    (2, 2, 128, 4, 9000, [130, 8700]),         # many splits: whole splits are padding
    (2, 3, 64, 8, 200, [5, 200]),              # 8-bit path; vf = pos: the new token only
    (144, 96, 128, 4, 96, None),               # opt-175b pairs, a mask that varies per sequence
])
def test_decode_attention_masked(batch, nh, d, bits, pos, vf):
    h = nh * d
    if vf is None:
        vf = [(7 * b) % (pos + 1) for b in range(batch)]
    vft = torch.tensor(vf, dtype=torch.int32, device="cuda")
    kh, vh = synth.kv_history(batch, nh, pos, d, pos + 1)
    cache = fq.FlexKVCache(batch, nh, d, pos + 2, bits, 64, valid_from=vft)
    cache.fill_from(kh.cuda(), vh.cuda())
    qkv = synth.activations((batch, 3 * h), pos + 2)
    qkv[:, :h] *= d ** -0.5
    g = qkv.cuda()
    o = torch.empty((batch, h), dtype=torch.float16, device="cuda")
    ws = torch.empty(max(16, fq.flex_decode_attention_ws_bytes(cache, batch, pos)), dtype=torch.uint8, device="cuda")
    fq.flex_decode_attention(cache, g[:, :h], g[:, h:2 * h], g[:, 2 * h:], 3 * h, o, batch, pos, ws)
    sync_status()
    rows = sorted(set([0, batch // 2, batch - 1]))
    oc = ol.KVCache(len(rows), nh, pos + 2, d, bits, 64)
    oc.store(kh.numpy()[rows], vh.numpy()[rows], 0)
    q = qkv.numpy()[rows]
    ref = ol.decode_attention(q[:, :h].reshape(-1, nh, d), q[:, h:2 * h].reshape(-1, nh, d),
                              q[:, 2 * h:].reshape(-1, nh, d), oc, pos, valid_from=[vf[r] for r in rows])
    assert_layer_close(o[rows], ref.reshape(len(rows), h), f"masked decode attention pos={pos}")


@pytest.mark.parametrize("batch,seq,nh,d,vf", [(2, 77, 3, 64, [0, 70]), (3, 200, 2, 128, [1, 64, 150]),
                                              (1, 130, 2, 64, [129])])
def test_prefill_attention_masked(batch, seq, nh, d, vf):
    h = nh * d
    qkv = synth.activations((batch, seq, 3 * h), seq + d)
    qkv[..., :h] *= d ** -0.5
    g = qkv.cuda()
    o = torch.full((batch, seq, h), float("nan"), dtype=torch.float16, device="cuda")
    vft = torch.tensor(vf, dtype=torch.int32, device="cuda")
    fq.flex_prefill_attention(g[..., :h], g[..., h:], g[..., 2 * h:], 3 * h, o, batch, seq, nh, d, valid_from=vft)
    sync_status()
    q = qkv.numpy()
    ref = ol.prefill_attention(q[..., :h].reshape(batch, seq, nh, d), q[..., h:2 * h].reshape(batch, seq, nh, d),
                               q[..., 2 * h:].reshape(batch, seq, nh, d), valid_from=vf)
    assert_layer_close(o, ref.reshape(batch, seq, h), f"masked prefill attention s={seq}")
    for b, v in enumerate(vf):                     # pad rows are exactly zero
        assert not o[b, :v].any()


@pytest.mark.parametrize("bits", [4, 8])
def test_layer_left_padded_prompts(bits):
    """opt-125m layer: 4 prompts padded on the left to 128 tokens (real lengths 128, 100,
    37, 1), prefill then 4 decode steps, against the oracle with the same padding."""
    cfg = dict(synth.WORKLOADS["opt-125m"])
    b, s, h, nh, d = 4, 128, cfg["h"], cfg["n_heads"], cfg["head_dim"]
    vf = [0, 28, 91, 127]
    raw = synth.layer_params(h, cfg["ffn"], 13)
    layer = fq.FlexLayer(raw, nh)
    PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
    W = ol.dequant_all(PQ)
    vft = torch.tensor(vf, dtype=torch.int32, device="cuda")
    cache = fq.FlexKVCache(b, nh, d, s + 4, bits, 64, valid_from=vft)
    ocache = ol.KVCache(b, nh, s + 4, d, bits, 64)
    x = synth.activations((b, s, h), 13)
    y = torch.empty((b, s, h), dtype=torch.float16, device="cuda")
    ws = torch.zeros(fq.flex_workspace_bytes(layer, b, s), dtype=torch.uint8, device="cuda")
    fq.flex_prefill_layer(layer, cache, x.cuda(), y, b, s, ws)
    sync_status()
    ref = ol.prefill_layer(x.numpy(), PQ, ocache, nh, W=W, valid_from=vf)
    assert_layer_close(y, ref, "padded prefill")
    wsd = torch.zeros(fq.flex_workspace_bytes(layer, b, 1), dtype=torch.uint8, device="cuda")
    for t in range(4):
        xd = synth.decode_inputs(b, h, t, 13)
        yd = torch.empty((b, h), dtype=torch.float16, device="cuda")
        fq.flex_decode_layer(layer, cache, xd.cuda(), yd, b, s + t, wsd)
        sync_status()
        refd = ol.decode_layer(xd.numpy(), PQ, ocache, s + t, nh, W=W, valid_from=vf)
        assert_layer_close(yd, refd, f"padded decode step {t}")
