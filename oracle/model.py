"""A whole synthetic OPT decoder for greedy generation - oracle; test infrastructure only.

Statement followed: the source-notes page «FlexGen» (PtirisNote), "Flex Opt" (the model is
an embedding, N transformer layers and an output head; OptLM.generate runs the
generation loop) and "Pytorch Backend" (opt_input_embed and opt_output_embed implement
the embedding layers); the walkthrough page «FlexGen 单 GPU 高吞吐大模型推理引擎：论文解读与源码实战指南», section 4.1 (the
generate API; do_sample=False is the deterministic, greedy choice).

Readings (the pages give no formulas for these; each is the plain OPT form):
  - input embedding: x = E^[token] + P[position], E the token table [V][h] compressed
    like the layer weights (4 bits, group 64 along h; E^ its fp16 dequantisation) and
    P a learned fp16 position table [max_pos][h]; the sum is rounded to fp16 once;
  - output head: the final LayerNorm, then logits = LN(h) E^T (the head shares the
    token table, as OPT's does);
  - greedy choice: the token with the largest logit, the lowest id among equal ones.
Arithmetic: float64 on the dequantised fp16 table, like oracle.layer.
"""
from __future__ import annotations

import numpy as np

from . import codec, layer

EMBED_CFG = dict(num_bits=4, group_size=64, group_dim=1)


def compress_table(E16):
    """Quantise the token table [V][h] (fp16) with the oracle codec (group 64 along h),
    as (codes, meta, shape) like oracle.layer's weights."""
    E16 = np.asarray(E16, np.float16)
    V, h = E16.shape
    codes = np.empty((V, h // 2), np.uint8)
    meta = np.empty((V, h // 64, 2), np.float16)
    for r0, r1 in layer._row_blocks(V, h):
        codes[r0:r1], meta[r0:r1] = codec.compress(E16[r0:r1], **EMBED_CFG)
    return codes, meta, E16.shape


def dequant_table(Eq):
    """E^ as fp16 [V][h]."""
    return layer.dequant_weight(Eq, dtype=np.float16)


def embed(tokens, positions, E_hat16, P16):
    """x [n][h] fp16 = fp16(E^[token] + P[position]) (exact sum, one rounding)."""
    t = np.asarray(tokens, np.int64)
    p = np.asarray(positions, np.int64)
    return (E_hat16[t].astype(np.float64) + P16[p].astype(np.float64)).astype(np.float16)


def logits(h16, lnf_g, lnf_b, E_hat16):
    """[n][V] float64 logits of the output head: LN(h; g, b) E^T."""
    a = layer.layer_norm(np.asarray(h16, np.float64), lnf_g, lnf_b)
    return layer.linear(a, E_hat16)


def greedy(logit_rows):
    """Token ids: the largest logit of each row, the lowest id among equal ones."""
    return np.argmax(np.asarray(logit_rows), axis=-1)          # numpy returns the first maximum


class Model:
    """n_layers OPT layers (oracle.layer on their dequantised weights), the compressed
    token table, the position table and the final LayerNorm."""

    def __init__(self, layers_raw, n_heads, E16, P16, lnf_g, lnf_b):
        self.nh = n_heads
        self.PQ = [layer.compress_weights(r) for r in layers_raw]
        self.W = [layer.dequant_all(q, dtype=np.float16 if r["w_o"].shape[0] >= 4096 else np.float64)
                  for q, r in zip(self.PQ, layers_raw)]
        self.Eq = compress_table(np.asarray(E16, np.float16))
        self.E_hat = dequant_table(self.Eq)
        self.P = np.asarray(P16, np.float16)
        self.lnf_g, self.lnf_b = np.asarray(lnf_g), np.asarray(lnf_b)

    def new_caches(self, batch, max_seq, head_dim):
        return [layer.KVCache(batch, self.nh, max_seq, head_dim) for _ in self.PQ]

    def prefill(self, prompt, caches):
        """prompt [b][s] token ids -> logits [b][V] of the last position (caches filled)."""
        b, s = prompt.shape
        x = embed(prompt.reshape(-1), np.tile(np.arange(s), b), self.E_hat, self.P).reshape(b, s, -1)
        for PQ, W, c in zip(self.PQ, self.W, caches):
            x = layer.prefill_layer(x, PQ, c, self.nh, W=W)
        return logits(x[:, -1], self.lnf_g, self.lnf_b, self.E_hat)

    def decode(self, tokens, pos, caches):
        """tokens [b] at position pos -> logits [b][V] (caches gain slot pos)."""
        x = embed(tokens, np.full(len(tokens), pos), self.E_hat, self.P)
        for PQ, W, c in zip(self.PQ, self.W, caches):
            x = layer.decode_layer(x, PQ, c, pos, self.nh, W=W)
        return logits(x, self.lnf_g, self.lnf_b, self.E_hat)
