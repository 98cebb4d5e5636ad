"""Layer parity at the OPT-30B and OPT-175B shapes (h 7168 / 12288, heads of 128),
through flex_prefill_layer and flex_decode_layer (C ABI).

These are the configurations of the pages' throughput setting (prompt 512, output 32,
effective batch 144; OPT-30B as 3 gpu-batches of 48). Decode batches above 32 run the
tcgen05 weight GEMM, whose QKV epilogue quantises the new token's key/value into cache
slot pos (store_cache), so these tests are the in-layer check of that path.

The GPU runs the whole batch; the oracle follows a few sampled sequences (sequences
are independent). No oracle input comes from the GPU.

Prefill: both sides run the prompt from the same seeded activations; outputs of the
sampled sequences within max|err| <= 1e-2 max|ref| + 1e-3; the cache slots the layer
wrote equal flexq_compress of its own fp16 keys/values bit for bit; and the cache is
within the quantiser's bound of the oracle's.

Decode: both sides start from one seeded fp16 key/value history, quantised into the
cache by flexq_compress (GPU) and by the oracle's codec - bit-identical by the codec's
own parity - and then run steps at the first (512) or the last (543) position of the
workload. A decode step that follows each side's own prefill is not compared at these
widths: the two prefills round the keys/values to fp16 differently in the last place,
the int4 codes then differ in about 0.5% of places, and at h 7168 the oracle's own
output moves by about 3x the tolerance under such a perturbation (an oracle-only
experiment), so the comparison would measure the rounding, not the kernels. The same
holds, on a smaller scale, for the one slot a decode step writes: at h 12288 the
second step moved by about 1.1x the tolerance when each side kept its own slot 512.
So each step checks the slot the layer wrote (flexq_compress of the layer's own fp16
key/value, bit for bit) and then overwrites it, on both sides, with the next slot of
the shared seeded history before the following step.
"""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import layer as ol
from _helpers import assert_layer_close, to_np, sync_status

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

MAX_SEQ = 544                        # prompt 512 + 32 decode steps


class _Model:
    """One synthetic layer: device parameters (compressed on the GPU) and the oracle's
    own compressed and dequantised copy of the same raw fp16 weights."""

    def __init__(self, name):
        cfg = dict(synth.WORKLOADS[name])
        self.cfg = cfg
        self.h, self.nh, self.d = cfg["h"], cfg["n_heads"], cfg["head_dim"]
        raw = synth.layer_params(cfg["h"], cfg["ffn"], cfg["seed"])
        self.layer = fq.FlexLayer(raw, self.nh)
        torch.cuda.synchronize()
        self.PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
        del raw
        self.W = ol.dequant_all(self.PQ, dtype=np.float16)


_models = {}


def _model(name):
    if name not in _models:
        _models.clear()              # one large layer on the host at a time
        _models[name] = _Model(name)
    return _models[name]


def _ws(layer, batch, seq):
    return torch.zeros(fq.flex_workspace_bytes(layer, batch, seq), dtype=torch.uint8, device="cuda")


def _ws_qkv(ws, batch, seq, h):
    """The layer's fp16 q|k|v [batch][seq][3h], the workspace region after LN1's output."""
    off = (batch * seq * h * 2 + 255) // 256 * 256
    return ws[off:off + batch * seq * 3 * h * 2].view(torch.float16).view(batch, seq, 3 * h)


def _check_cache_slots(cache, ws, batch, seq, pos0, h, nh, d):
    """Slots [pos0, pos0 + seq) of every sequence = flexq_compress of the layer's own
    fp16 keys/values, bit for bit."""
    qkv = _ws_qkv(ws, batch, seq, h)
    for sec, (codes, meta) in enumerate(((cache.k_codes, cache.k_meta), (cache.v_codes, cache.v_meta))):
        t16 = qkv[..., (1 + sec) * h:(2 + sec) * h].reshape(batch, seq, nh, d).permute(0, 2, 1, 3).contiguous()
        c, m = fq.flexq_compress(t16, cache.cfg)
        sync_status()
        assert torch.equal(codes[:batch, :, pos0:pos0 + seq], c), f"cache codes ({'kv'[sec]}) differ"
        assert torch.equal(meta[:batch, :, pos0:pos0 + seq], m), f"cache metadata ({'kv'[sec]}) differ"


def _check_prefill_cache_bound(cache, ocache, rows, seq, nh, d):
    """Dequantised GPU cache of the sampled sequences vs the oracle's: within two
    quantisation steps of the group range (keys/values differ by GEMM rounding only)."""
    idx = torch.tensor(rows, device="cuda")
    for codes, meta, which in ((cache.k_codes, cache.k_meta, 0), (cache.v_codes, cache.v_meta, 1)):
        c = codes.index_select(0, idx)[:, :, :seq].contiguous()
        m = meta.index_select(0, idx)[:, :, :seq].contiguous()
        g = to_np(fq.flexq_decompress(c, m, (len(rows), nh, seq, d), cache.cfg)).astype(np.float64)
        sync_status()
        ref = ocache.load(seq)[which]
        rng = ref.max(-1, keepdims=True) - ref.min(-1, keepdims=True)
        assert np.all(np.abs(g - ref) <= 2 * rng / 15 + 2e-2), "prefill cache outside the quantiser bound"


@pytest.mark.parametrize("name,batch,rows,prompt", [
    ("opt-30b", 48, [0, 47], 512),               # one gpu-batch of 48
    ("opt-175b", 144, [0, 143], 543),            # the whole batch, the longest prompt
])
def test_large_layer_prefill(name, batch, rows, prompt):
    M = _model(name)
    h, nh, d, seed = M.h, M.nh, M.d, M.cfg["seed"]
    cache = fq.FlexKVCache(batch, nh, d, MAX_SEQ)
    ocache = ol.KVCache(len(rows), nh, MAX_SEQ, d)
    x = synth.activations((batch, prompt, h), seed)
    y = torch.empty((batch, prompt, h), dtype=torch.float16, device="cuda")
    ws = _ws(M.layer, batch, prompt)
    fq.flex_prefill_layer(M.layer, cache, x.cuda(), y, batch, prompt, ws)
    sync_status()
    _check_cache_slots(cache, ws, batch, prompt, 0, h, nh, d)
    del ws
    ref = ol.prefill_layer(x.numpy()[rows], M.PQ, ocache, nh, W=M.W)
    assert_layer_close(y[rows], ref, f"{name} prefill b={batch} s={prompt} (sampled)")
    _check_prefill_cache_bound(cache, ocache, rows, prompt, nh, d)
    del y
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name,batch,rows,pos,steps", [
    ("opt-30b", 48, [0, 47], 512, 2),            # one gpu-batch of 48: the first decode steps
    ("opt-30b", 144, [0, 71, 143], 543, 1),      # 144 in one call: the last decode step
    ("opt-175b", 144, [0, 143], 512, 2),         # first steps
    ("opt-175b", 144, [0, 143], 543, 1),         # last step (slot 543 of 544)
])
def test_large_layer_decode(name, batch, rows, pos, steps):
    M = _model(name)
    h, nh, d, seed = M.h, M.nh, M.d, M.cfg["seed"]
    n_hist = pos + steps - 1                      # the shared history also supplies later steps' slots
    kh, vh = synth.kv_history(batch, nh, n_hist, d, seed + 50, device="cuda")
    cache = fq.FlexKVCache(batch, nh, d, MAX_SEQ)
    cache.fill_from(kh[:, :, :pos], vh[:, :, :pos])
    ocache = ol.KVCache(len(rows), nh, MAX_SEQ, d)
    ocache.store(to_np(kh[rows, :, :pos]), to_np(vh[rows, :, :pos]), 0)
    k_next, v_next = kh[:, :, pos:].contiguous(), vh[:, :, pos:].contiguous()
    del kh, vh
    torch.cuda.empty_cache()
    wsd = _ws(M.layer, batch, 1)
    for t in range(steps):
        if t > 0:                                 # slot pos + t - 1 from the shared history, both sides
            sl = slice(t - 1, t)
            for src, codes, meta in ((k_next[:, :, sl], cache.k_codes, cache.k_meta),
                                     (v_next[:, :, sl], cache.v_codes, cache.v_meta)):
                c, m = fq.flexq_compress(src.contiguous(), cache.cfg)
                codes[:, :, pos + t - 1:pos + t].copy_(c)
                meta[:, :, pos + t - 1:pos + t].copy_(m)
            ocache.store(to_np(k_next[rows, :, sl]), to_np(v_next[rows, :, sl]), pos + t - 1)
        xd = synth.decode_inputs(batch, h, t, seed)
        yd = torch.empty((batch, h), dtype=torch.float16, device="cuda")
        fq.flex_decode_layer(M.layer, cache, xd.cuda(), yd, batch, pos + t, wsd)
        sync_status()
        _check_cache_slots(cache, wsd, batch, 1, pos + t, h, nh, d)
        refd = ol.decode_layer(xd.numpy()[rows], M.PQ, ocache, pos + t, nh, W=M.W)
        assert_layer_close(yd[rows], refd, f"{name} decode b={batch} pos={pos + t} (sampled)")
