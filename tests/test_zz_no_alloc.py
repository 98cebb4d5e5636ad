"""flex_decode_attention_noalloc: decode attention for callers that cannot allocate
device memory (a plain C host program with no device allocator, or a path that must
make progress after an out-of-memory error). Its split-KV partials live in a scratch
buffer compiled into the library instead of a caller workspace.

The same kernels and the same split plan run in both entry points, so the output must
be bit-identical to flex_decode_attention's; it is also checked against the oracle's
decode attention. The cases make the kernels really use the scratch: the 8-bit path
always writes partials (about 7.2 MB of them at 144 sequences x 96 heads of 128), and
a few (sequence, head) pairs with a long history split their keys over many CTAs. A
call that needs many splits runs right after one that wrote fewer, so a partial left
over from an earlier call would be caught.

The file name sorts last so that the entry point is also exercised after every other
GPU test of the session has run; it passes on its own in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import layer as ol
from _helpers import assert_layer_close, to_np, sync_status

pytestmark = pytest.mark.gpu


def _inputs(batch, nh, d, bits, gs, pos, seed, max_seq=None):
    h = nh * d
    cache = fq.FlexKVCache(batch, nh, d, max_seq or pos + 2, bits, gs)
    kh = vh = None
    if pos > 0:
        kh, vh = synth.kv_history(batch, nh, pos, d, seed, device="cuda")
        cache.fill_from(kh, vh)
    qkv = synth.activations((batch, 3 * h), seed + 1, device="cuda")
    qkv[:, :h] *= d ** -0.5
    return cache, qkv, kh, vh


def _oracle(qkv, kh, vh, rows, nh, d, bits, gs, pos, max_seq):
    h = nh * d
    oc = ol.KVCache(len(rows), nh, max_seq, d, bits, gs)
    if pos > 0:
        oc.store(to_np(kh[rows]), to_np(vh[rows]), 0)
    q = to_np(qkv[rows])
    return ol.decode_attention(q[:, :h].reshape(-1, nh, d), q[:, h:2 * h].reshape(-1, nh, d),
                               q[:, 2 * h:].reshape(-1, nh, d), oc, pos).reshape(len(rows), h)


def _workspace_reference(cache, qkv, batch, pos, h):
    need = fq.flex_decode_attention_ws_bytes(cache, batch, pos)
    assert need <= fq.FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES
    ws = torch.empty(max(16, need), dtype=torch.uint8, device="cuda")
    ref = torch.empty((batch, h), dtype=torch.float16, device="cuda")
    fq.flex_decode_attention(cache, qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:], 3 * h, ref, batch, pos, ws)
    sync_status()
    return ref, need


@pytest.mark.parametrize("batch,nh,d,bits,gs,pos,min_scratch", [
    (144, 96, 128, 8, 64, 33, 7_000_000),  # opt-175b shape, 8-bit cache: ~7.2 MB of partials
    (2, 4, 128, 4, 64, 9000, 200 << 10),  # 8 pairs, long history: 71 splits per pair
    (32, 32, 64, 4, 64, 543, 0),          # opt-1.3b decode shape: one split, no partials read
    (4, 12, 64, 4, 64, 0, 0),             # empty history: fresh key/value only
    (2, 4, 128, 8, 32, 77, 0),            # 8-bit cache, group 32
])
def test_noalloc_bit_identical_to_workspace_entry(batch, nh, d, bits, gs, pos, min_scratch):
    h = nh * d
    cache, qkv, kh, vh = _inputs(batch, nh, d, bits, gs, pos, seed=900 + pos)
    ref, need = _workspace_reference(cache, qkv, batch, pos, h)
    assert need >= min_scratch
    rows = [0, batch - 1]
    assert_layer_close(ref[rows], _oracle(qkv, kh, vh, rows, nh, d, bits, gs, pos, pos + 2), "workspace entry")
    for call in range(2):
        o = torch.full((batch, h), float("nan"), dtype=torch.float16, device="cuda")
        fq.flex_decode_attention_noalloc(cache, qkv[:, :h], qkv[:, h:2 * h], qkv[:, 2 * h:], 3 * h, o, batch, pos)
        sync_status()
        assert torch.equal(o, ref), f"no-alloc decode attention differs from the workspace entry (call {call + 1})"


def test_more_splits_after_fewer_reads_no_stale_partials():
    """Call A (one sequence, 300 keys: 3 splits) fills the start of the scratch; call B
    (two sequences, 9000 keys: 71 splits per pair) then needs partials at offsets A
    never wrote and at ones it did. B must equal the workspace entry bit for bit."""
    nh, d = 4, 128
    h = nh * d
    cache_a, qkv_a, _, _ = _inputs(1, nh, d, 4, 64, 300, seed=5)
    oa = torch.empty((1, h), dtype=torch.float16, device="cuda")
    fq.flex_decode_attention_noalloc(cache_a, qkv_a[:, :h], qkv_a[:, h:2 * h], qkv_a[:, 2 * h:], 3 * h, oa, 1, 300)
    sync_status()
    ref_a, _ = _workspace_reference(cache_a, qkv_a, 1, 300, h)
    assert torch.equal(oa, ref_a)
    cache_b, qkv_b, _, _ = _inputs(2, nh, d, 4, 64, 9000, seed=6)
    ref_b, need_b = _workspace_reference(cache_b, qkv_b, 2, 9000, h)
    assert need_b > fq.flex_decode_attention_ws_bytes(cache_a, 1, 300)
    ob = torch.empty((2, h), dtype=torch.float16, device="cuda")
    fq.flex_decode_attention_noalloc(cache_b, qkv_b[:, :h], qkv_b[:, h:2 * h], qkv_b[:, 2 * h:], 3 * h, ob, 2, 9000)
    sync_status()
    assert torch.equal(ob, ref_b)


def test_noalloc_rejects_problem_beyond_scratch():
    """A problem whose partials exceed the built-in buffer is refused before launch."""
    batch, nh, d, pos = 200, 96, 128, 5          # 19200 pairs x 130 fp32 > 8 MiB
    cache, qkv, _, _ = _inputs(batch, nh, d, 4, 64, pos, seed=31)
    h = nh * d
    assert fq.flex_decode_attention_ws_bytes(cache, batch, pos) > fq.FLEX_DECODE_ATTENTION_STATIC_MAX_BYTES
    o = torch.zeros((batch, h), dtype=torch.float16, device="cuda")
    with pytest.raises(fq.FlexError) as err:
        fq.flex_decode_attention_noalloc(cache, qkv[:, :h], qkv[:, h:], qkv[:, 2 * h:], 3 * h, o, batch, pos)
    assert err.value.code == fq.FLEX_ERR_SCRATCH_LIMIT
    sync_status()
    assert not o.any()
