"""flex_prefill_layer_batches / flex_decode_layer_batches: several gpu-batches, each with
its own KV cache, through one layer with a single pass over the weights (the pages'
gpu_batch_size x num_gpu_batches block). Checked against the oracle run per gpu-batch
with its own cache, and against separate single-batch layer calls.
Tolerance: max|err| <= 1e-2 max|ref| + 1e-3."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import layer as ol
from _helpers import assert_layer_close, sync_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nb,b,s,steps", [(3, 4, 33, 3),     # 12 activation rows: the GEMV path
                                          (3, 16, 20, 2),    # 48 rows: the tcgen05 GEMM path
                                          (2, 3, 1, 1)])     # one-token prompts
def test_batches_match_oracle_per_gpu_batch(nb, b, s, steps):
    cfg = dict(synth.WORKLOADS["opt-125m"])
    h, nh, d = cfg["h"], cfg["n_heads"], cfg["head_dim"]
    raw = synth.layer_params(h, cfg["ffn"], 21)
    layer = fq.FlexLayer(raw, nh)
    PQ = ol.compress_weights({k: v.numpy() for k, v in raw.items()})
    W = ol.dequant_all(PQ)
    max_seq = s + steps
    caches = [fq.FlexKVCache(b, nh, d, max_seq) for _ in range(nb)]
    ocaches = [ol.KVCache(b, nh, max_seq, d) for _ in range(nb)]
    x = synth.activations((nb, b, s, h), 21)
    y = torch.empty((nb, b, s, h), dtype=torch.float16, device="cuda")
    ws = torch.zeros(fq.flex_workspace_bytes(layer, nb * b, s), dtype=torch.uint8, device="cuda")
    fq.flex_prefill_layer_batches(layer, caches, x.cuda(), y, b, s, ws)
    sync_status()
    for c in range(nb):
        ref = ol.prefill_layer(x[c].numpy(), PQ, ocaches[c], nh, W=W)
        assert_layer_close(y[c], ref, f"prefill gpu-batch {c}")
    wsd = torch.zeros(fq.flex_workspace_bytes(layer, nb * b, 1), dtype=torch.uint8, device="cuda")
    for t in range(steps):
        xd = synth.decode_inputs(nb * b, h, t, 21).view(nb, b, h)
        yd = torch.empty((nb, b, h), dtype=torch.float16, device="cuda")
        fq.flex_decode_layer_batches(layer, caches, xd.cuda(), yd, b, s + t, wsd)
        sync_status()
        for c in range(nb):
            refd = ol.decode_layer(xd[c].numpy(), PQ, ocaches[c], s + t, nh, W=W)
            assert_layer_close(yd[c], refd, f"decode step {t} gpu-batch {c}")


def test_batches_equal_separate_calls():
    """The block schedule and one call per gpu-batch differ only in summation order;
    their caches (slots written by the decode step) agree up to that too."""
    cfg = dict(synth.WORKLOADS["opt-125m"])
    h, nh, d = cfg["h"], cfg["n_heads"], cfg["head_dim"]
    nb, b, pos = 3, 8, 40
    raw = synth.layer_params(h, cfg["ffn"], 22)
    layer = fq.FlexLayer(raw, nh)
    kh, vh = synth.kv_history(nb * b, nh, pos, d, 22, device="cuda")
    ca = [fq.FlexKVCache(b, nh, d, pos + 1) for _ in range(nb)]
    cb = [fq.FlexKVCache(b, nh, d, pos + 1) for _ in range(nb)]
    for c in range(nb):
        ca[c].fill_from(kh[c * b:(c + 1) * b], vh[c * b:(c + 1) * b])
        cb[c].fill_from(kh[c * b:(c + 1) * b], vh[c * b:(c + 1) * b])
    x = synth.decode_inputs(nb * b, h, 0, 22, device="cuda")
    ya = torch.empty_like(x)
    fq.flex_decode_layer_batches(layer, ca, x, ya, b, pos,
                                 torch.zeros(fq.flex_workspace_bytes(layer, nb * b, 1), dtype=torch.uint8,
                                             device="cuda"))
    yb = torch.empty_like(x)
    ws = torch.zeros(fq.flex_workspace_bytes(layer, b, 1), dtype=torch.uint8, device="cuda")
    for c in range(nb):
        fq.flex_decode_layer(layer, cb[c], x[c * b:(c + 1) * b], yb[c * b:(c + 1) * b], b, pos, ws)
    sync_status()
    assert_layer_close(ya, yb.double().cpu().numpy(), "block schedule vs separate calls")
    for c in range(nb):
        kd = (ca[c].k_codes[:, :, pos].int() & 15) - (cb[c].k_codes[:, :, pos].int() & 15)
        assert int(kd.abs().max()) <= 1


def test_batches_bad_args():
    cfg = dict(synth.WORKLOADS["opt-125m"])
    raw = synth.layer_params(cfg["h"], cfg["ffn"], 1)
    layer = fq.FlexLayer(raw, cfg["n_heads"])
    caches = [fq.FlexKVCache(2, cfg["n_heads"], cfg["head_dim"], 8), fq.FlexKVCache(2, cfg["n_heads"], cfg["head_dim"], 9)]
    x = torch.zeros((2, 2, cfg["h"]), dtype=torch.float16, device="cuda")
    y = torch.zeros_like(x)
    ws = torch.zeros(fq.flex_workspace_bytes(layer, 4, 1), dtype=torch.uint8, device="cuda")
    with pytest.raises(fq.FlexError) as e:                 # caches of different lengths
        fq.flex_decode_layer_batches(layer, caches, x, y, 2, 0, ws)
    assert e.value.code == fq.FLEX_ERR_SHAPE
    with pytest.raises(fq.FlexError) as e:                 # more than 8 gpu-batches
        fq.flex_decode_layer_batches(layer, [caches[0]] * 9, x, y, 2, 0, ws)
    assert e.value.code == fq.FLEX_ERR_INVALID_ARG
