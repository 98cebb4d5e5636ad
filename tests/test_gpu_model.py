"""The whole synthetic model around the layers - input embedding (flex_embed), output
head with the greedy choice (flex_lm_head_argmax) and a greedy generation loop through
two OPT-125M-shaped layers - against oracle.model.

The embedding is bit-exact. Logits: max|err| <= 1e-2 max|ref| + 1e-3. A greedy id is a
decision taken on floating point, so it is compared where it is unique: the oracle's
logit of the GPU's id must be within the logit tolerance of the oracle's largest one,
and in the generation loop the two sequences must agree token for token until the
oracle meets a near tie (top two logits closer than twice the tolerance)."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import model as om
from _helpers import assert_bits_equal, assert_layer_close, layer_tolerance, to_np, sync_status

pytestmark = pytest.mark.gpu

V = synth.OPT_VOCAB
V_PAD = (V + 255) // 256 * 256


def _table(h, max_pos, seed, vocab=V, vocab_pad=V_PAD):
    mp = synth.model_params(vocab, h, max_pos, seed, vocab_pad)
    E = fq.CompressedWeight(mp["E"].cuda())
    return mp, E


def test_embed_bit_exact_and_range_check():
    h, max_pos, n = 768, 64, 37
    mp, E = _table(h, max_pos, 1)
    tok = synth.token_ids((n,), V, 2)
    pos = synth.token_ids((n,), max_pos, 3)
    x = fq.flex_embed(E, V, mp["P"].cuda(), tok.cuda(), pos.cuda())
    sync_status()
    E_hat = om.dequant_table(om.compress_table(mp["E"].numpy()))
    assert_bits_equal(x, om.embed(tok.numpy(), pos.numpy(), E_hat, mp["P"].numpy()), "embedding")
    bad = torch.tensor([V + 5, -1], dtype=torch.int32, device="cuda")
    fq.flex_embed(E, V, mp["P"].cuda(), bad, torch.zeros(2, dtype=torch.int32, device="cuda"))
    assert fq.flex_get_status() == fq.FLEX_ERR_INVALID_ARG


def _check_choice(gpu_ids, ref_logits, what):
    tol = layer_tolerance(ref_logits)
    best = ref_logits.max(-1)
    got = ref_logits[np.arange(len(gpu_ids)), gpu_ids]
    assert np.all(got >= best - tol), f"{what}: greedy ids not within tolerance of the best logit"


@pytest.mark.parametrize("n", [1, 5, 48])
def test_head_logits_and_greedy_choice(n):
    h = 768
    mp, E = _table(h, 8, 4)
    x = synth.activations((n, h), 5)
    ws = torch.zeros(fq.flex_lm_head_ws_bytes(E, V, n, True), dtype=torch.uint8, device="cuda")
    logits = torch.empty((n, V_PAD), dtype=torch.float16, device="cuda")
    ids = fq.flex_lm_head_argmax(E, V, mp["lnf_g"].cuda(), mp["lnf_b"].cuda(), x.cuda(), ws, logits=logits)
    sync_status()
    E_hat = om.dequant_table(om.compress_table(mp["E"].numpy()))
    ref = om.logits(x.numpy(), mp["lnf_g"].numpy(), mp["lnf_b"].numpy(), E_hat[:V])
    assert_layer_close(logits[:, :V], ref, "head logits")
    g = to_np(ids).astype(np.int64)
    _check_choice(g, ref, "head")
    # the choice is the first maximum of the kernel's own fp16 logits
    assert np.array_equal(g, np.argmax(to_np(logits[:, :V]).astype(np.float32), axis=-1))
    # without a logits buffer: the same ids
    ws2 = torch.zeros(fq.flex_lm_head_ws_bytes(E, V, n, False), dtype=torch.uint8, device="cuda")
    ids2 = fq.flex_lm_head_argmax(E, V, mp["lnf_g"].cuda(), mp["lnf_b"].cuda(), x.cuda(), ws2)
    sync_status()
    assert torch.equal(ids, ids2)


def test_greedy_generation_two_layers():
    cfg = dict(synth.WORKLOADS["opt-125m"])
    h, nh, d, ffn = cfg["h"], cfg["n_heads"], cfg["head_dim"], cfg["ffn"]
    b, s, steps, L = 4, 12, 6, 2
    max_seq = s + steps
    raws = [synth.layer_params(h, ffn, 30 + l) for l in range(L)]
    mp, E = _table(h, max_seq, 6)
    layers = [fq.FlexLayer(r, nh) for r in raws]
    caches = [fq.FlexKVCache(b, nh, d, max_seq) for _ in range(L)]
    P, g, bb = mp["P"].cuda(), mp["lnf_g"].cuda(), mp["lnf_b"].cuda()
    prompt = synth.token_ids((b, s), V, 7)
    # GPU loop
    x = fq.flex_embed(E, V, P, prompt.reshape(-1).cuda(), torch.arange(s, dtype=torch.int32).repeat(b).cuda())
    x = x.view(b, s, h)
    ws = torch.zeros(fq.flex_workspace_bytes(layers[0], b, s), dtype=torch.uint8, device="cuda")
    for l in range(L):
        y = torch.empty_like(x)
        fq.flex_prefill_layer(layers[l], caches[l], x, y, b, s, ws)
        x = y
    hws = torch.zeros(fq.flex_lm_head_ws_bytes(E, V, b, False), dtype=torch.uint8, device="cuda")
    ids = fq.flex_lm_head_argmax(E, V, g, bb, x[:, -1].contiguous(), hws)
    gpu_tokens = [to_np(ids).astype(np.int64)]
    wsd = torch.zeros(fq.flex_workspace_bytes(layers[0], b, 1), dtype=torch.uint8, device="cuda")
    for t in range(steps - 1):
        pos = s + t
        x = fq.flex_embed(E, V, P, ids, torch.full((b,), pos, dtype=torch.int32, device="cuda"))
        for l in range(L):
            y = torch.empty_like(x)
            fq.flex_decode_layer(layers[l], caches[l], x, y, b, pos, wsd)
            x = y
        ids = fq.flex_lm_head_argmax(E, V, g, bb, x, hws)
        gpu_tokens.append(to_np(ids).astype(np.int64))
    sync_status()
    # oracle loop (its own greedy choices)
    m = om.Model([{k: v.numpy() for k, v in r.items()} for r in raws], nh, mp["E"].numpy()[:V], mp["P"].numpy(),
                 mp["lnf_g"].numpy(), mp["lnf_b"].numpy())
    oc = m.new_caches(b, max_seq, d)
    lg = m.prefill(prompt.numpy().astype(np.int64), oc)
    live = np.ones(b, bool)                        # sequences still compared
    compared = 0
    for t in range(steps):
        tol = layer_tolerance(lg)
        top2 = np.sort(lg, axis=-1)[:, -2:]
        live &= (top2[:, 1] - top2[:, 0]) > 2 * tol
        ref_ids = om.greedy(lg)
        assert np.array_equal(gpu_tokens[t][live], ref_ids[live]), (t, gpu_tokens[t], ref_ids)
        compared += int(live.sum())
        if t + 1 < steps:
            lg = m.decode(ref_ids, s + t, oc)
    assert compared >= b, "every sequence met a near tie at once: nothing was compared"
