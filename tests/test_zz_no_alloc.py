"""flex_decode_attention_noalloc (partials in the library's built-in scratch) against
flex_decode_attention (caller workspace) on the same inputs, called twice in a row.

The file name sorts last so that the entry point is also exercised after every other
GPU test of the session has run (and with it, the library's other kernels); it passes
on its own in a fresh process as well.
"""
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from _helpers import assert_layer_close, sync_status

pytestmark = pytest.mark.gpu


def _inputs(batch, nh, d, bits, gs, pos, seed):
    h = nh * d
    cache = fq.FlexKVCache(batch, nh, d, pos + 2, bits, gs)
    if pos > 0:
        kh, vh = synth.kv_history(batch, nh, pos, d, seed, device="cuda")
        cache.fill_from(kh, vh)
    qkv = synth.activations((batch, 3 * h), seed + 1, device="cuda")
    qkv[:, :h] *= d ** -0.5
    return cache, qkv


@pytest.mark.parametrize("batch,nh,d,bits,gs,pos", [
    (32, 32, 64, 4, 64, 543),     # opt-1.3b decode shape, 4-bit cache
    (4, 12, 64, 4, 64, 0),        # empty history: fresh key/value only
    (3, 5, 128, 4, 64, 130),      # ragged split of 130 keys
    (2, 4, 128, 8, 32, 77),       # 8-bit cache, group 32
    (144, 96, 128, 4, 64, 33),    # opt-175b shape: largest scratch of the workloads
])
def test_noalloc_matches_workspace_entry(batch, nh, d, bits, gs, pos):
    h = nh * d
    cache, qkv = _inputs(batch, nh, d, bits, gs, pos, seed=900 + pos)
    q, kn, vn = qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:]
    need = fq.flex_decode_attention_ws_bytes(cache, batch, pos)
    assert 0 < need <= fq.FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    ref = torch.empty((batch, h), dtype=torch.float16, device="cuda")
    fq.flex_decode_attention(cache, q, kn, vn, 3 * h, ref, batch, pos, ws)
    sync_status()
    expected = ref.double().cpu().numpy()
    for call in range(2):
        o = torch.full((batch, h), float("nan"), dtype=torch.float16, device="cuda")
        fq.flex_decode_attention_noalloc(cache, q, kn, vn, 3 * h, o, batch, pos)
        sync_status()
        assert_layer_close(o, expected, f"no-alloc decode attention, call {call + 1}")


def test_noalloc_rejects_problem_beyond_scratch():
    """A problem whose partials exceed the built-in buffer is refused before launch."""
    batch, nh, d, pos = 200, 96, 128, 5          # 19200 pairs x 130 fp32 > 8 MiB
    cache, qkv = _inputs(batch, nh, d, 4, 64, pos, seed=31)
    h = nh * d
    assert fq.flex_decode_attention_ws_bytes(cache, batch, pos) > fq.FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES
    o = torch.zeros((batch, h), dtype=torch.float16, device="cuda")
    with pytest.raises(fq.FlexError) as err:
        fq.flex_decode_attention_noalloc(cache, qkv[:, :h], qkv[:, h:], qkv[:, 2 * h:], 3 * h, o, batch, pos)
    assert err.value.code == fq.FLEX_ERR_SCRATCH_LIMIT
    sync_status()
    assert not o.any()
