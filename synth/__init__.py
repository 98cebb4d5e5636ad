"""Seeded synthetic inputs shared by the oracle side and the CUDA side of every test
and of the benchmark.

This module only draws random numbers and arranges them into the shapes, value
distributions and structure of the workloads. It holds none of the method's
arithmetic: no quantisation, no layer math. Both sides of a parity check receive
the very same tensors from here (one copy goes to the host oracle, one to the
device), so any disagreement comes from the arithmetic, never from the inputs.

Workloads (OPT decoder-layer shapes, FlexGen's "High-throughput Generative
Inference of Large Language Models with a Single GPU" setting of prompt 512 /
output 32, and the group-wise 4-bit compression configuration of FlexGen's
compression module: 4 bits, group 64):

  opt-125m : h=768,   12 heads x 64,  ffn 3072,  batch 4,   prompt 128, 8 decode steps
  opt-1.3b : h=2048,  32 heads x 64,  ffn 8192,  batch 32,  prompt 512, 32 decode steps
  opt-30b  : h=7168,  56 heads x 128, ffn 28672, batch 144 (3 gpu-batches of 48), 512 + 32
  opt-175b : h=12288, 96 heads x 128, ffn 49152, batch 144, 512 + 32, 4 distinct layers
  codec    : fp16 [R, 4096] tensors of 1 MB .. 4 GB, N(0,1) with 0.1% outliers x50,
             1% constant groups and one all-zero group
"""
from __future__ import annotations

import math

import torch

WORKLOADS = {
    "opt-125m": dict(h=768, n_heads=12, head_dim=64, ffn=3072, batch=4, prompt=128,
                     decode_steps=8, layers=1, seed=1),
    "opt-1.3b": dict(h=2048, n_heads=32, head_dim=64, ffn=8192, batch=32, prompt=512,
                     decode_steps=32, layers=24, seed=2),
    "opt-30b": dict(h=7168, n_heads=56, head_dim=128, ffn=28672, batch=144, gpu_batch=48,
                    prompt=512, decode_steps=32, layers=1, seed=3),
    "opt-175b": dict(h=12288, n_heads=96, head_dim=128, ffn=49152, batch=144, prompt=512,
                     decode_steps=32, layers=4, seed=4),
}

WEIGHT_STD = 0.02     # weights N(0, 0.02)
PARAM_STD = 0.02      # biases N(0, 0.02); LayerNorm gamma 1 + N(0, 0.02), beta N(0, 0.02)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_f16(shape, seed: int, std: float = 1.0, mean: float = 0.0, device="cpu") -> torch.Tensor:
    """N(mean, std^2) drawn in fp32 and rounded once to fp16."""
    g = _gen(seed, device)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    if mean != 0.0:
        t.add_(mean)
    return t.to(torch.float16)


def layer_params(h: int, ffn: int, seed: int, device="cpu") -> dict:
    """Raw fp16 parameters of one OPT decoder layer (weights stored [out][in]).

    The fused QKV weight stacks the query, key and value projections as rows
    [q; k; v]; inside each block, output feature = head * head_dim + j.
    """
    s = int(seed) * 1000
    p = {
        "w_qkv": normal_f16((3 * h, h), s + 1, WEIGHT_STD, device=device),
        "w_o": normal_f16((h, h), s + 2, WEIGHT_STD, device=device),
        "w_fc1": normal_f16((ffn, h), s + 3, WEIGHT_STD, device=device),
        "w_fc2": normal_f16((h, ffn), s + 4, WEIGHT_STD, device=device),
        "b_qkv": normal_f16((3 * h,), s + 5, PARAM_STD, device=device),
        "b_o": normal_f16((h,), s + 6, PARAM_STD, device=device),
        "b_fc1": normal_f16((ffn,), s + 7, PARAM_STD, device=device),
        "b_fc2": normal_f16((h,), s + 8, PARAM_STD, device=device),
        "ln1_g": normal_f16((h,), s + 9, PARAM_STD, mean=1.0, device=device),
        "ln1_b": normal_f16((h,), s + 10, PARAM_STD, device=device),
        "ln2_g": normal_f16((h,), s + 11, PARAM_STD, mean=1.0, device=device),
        "ln2_b": normal_f16((h,), s + 12, PARAM_STD, device=device),
    }
    return p


OPT_VOCAB = 50272     # token ids of the OPT family's tokenizer


def model_params(vocab: int, h: int, max_pos: int, seed: int, vocab_pad: int = None, device="cpu") -> dict:
    """Token table E [vocab_pad][h] (rows >= vocab zero: padding no token uses), position
    table P [max_pos][h], both N(0, 0.02) fp16, and the final LayerNorm's gain
    1 + N(0, 0.02) and bias N(0, 0.02)."""
    s = int(seed) * 1000 + 900
    vocab_pad = vocab_pad or vocab
    E = torch.zeros((vocab_pad, h), dtype=torch.float16, device=device)
    E[:vocab] = normal_f16((vocab, h), s + 1, WEIGHT_STD, device=device)
    return {"E": E, "P": normal_f16((max_pos, h), s + 2, WEIGHT_STD, device=device),
            "lnf_g": normal_f16((h,), s + 3, PARAM_STD, mean=1.0, device=device),
            "lnf_b": normal_f16((h,), s + 4, PARAM_STD, device=device)}


def token_ids(shape, vocab: int, seed: int, device="cpu") -> torch.Tensor:
    """Uniform token ids in [0, vocab), int32."""
    g = _gen(int(seed) * 1000 + 950, device)
    return torch.randint(0, int(vocab), tuple(shape), generator=g, device=device, dtype=torch.int64).to(torch.int32)


def activations(shape, seed: int, device="cpu") -> torch.Tensor:
    """Layer input activations, N(0, 1) fp16."""
    return normal_f16(shape, int(seed) * 1000 + 500, 1.0, device=device)


def decode_inputs(batch: int, h: int, step: int, seed: int, device="cpu") -> torch.Tensor:
    """Fresh N(0, 1) input of decode step `step` (a synthetic layer has no LM feedback)."""
    return normal_f16((batch, h), int(seed) * 1000 + 600 + int(step), 1.0, device=device)


def kv_history(batch: int, n_heads: int, length: int, head_dim: int, seed: int, device="cpu"):
    """fp16 key and value histories [batch][n_heads][length][head_dim], N(0, 1)."""
    k = normal_f16((batch, n_heads, length, head_dim), int(seed) * 1000 + 700, 1.0, device=device)
    v = normal_f16((batch, n_heads, length, head_dim), int(seed) * 1000 + 701, 1.0, device=device)
    return k, v


def codec_tensor(shape, group_dim: int, group_size: int, seed: int, device="cpu",
                 outlier_p: float = 1e-3, outlier_scale: float = 50.0,
                 const_group_p: float = 0.01) -> torch.Tensor:
    """fp16 tensor for the compression sweep.

    Values N(0, 1); a Bernoulli(outlier_p) subset is multiplied by outlier_scale;
    about const_group_p of the groups (runs of group_size along group_dim) are set
    to a single N(0, 1) draw each, and the first group is all zeros.
    """
    shape = tuple(int(d) for d in shape)
    nd = len(shape)
    gd = group_dim % nd
    g = _gen(seed, device)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    mask = torch.rand(shape, generator=g, device=device) < outlier_p
    x = torch.where(mask, x * outlier_scale, x)
    # group view: move the group dim last and split it into (ng, gs)
    xm = x.movedim(gd, -1)
    lead = xm.shape[:-1]
    ng = xm.shape[-1] // group_size
    xg = xm.reshape(*lead, ng, group_size)
    n_groups = xg.numel() // group_size
    const = torch.rand(xg.shape[:-1], generator=g, device=device) < const_group_p
    cval = torch.randn(xg.shape[:-1], generator=g, device=device)
    xg = torch.where(const.unsqueeze(-1), cval.unsqueeze(-1).expand_as(xg), xg)
    flat = xg.reshape(n_groups, group_size)
    flat[0].zero_()
    x = xg.reshape(*lead, ng * group_size).movedim(-1, gd)
    return x.to(torch.float16).contiguous()


def codec_rows_for_bytes(nbytes: int, cols: int = 4096) -> int:
    """Rows of a fp16 [R, cols] tensor holding nbytes."""
    return max(1, nbytes // (2 * cols))


def ceil_div(a: int, b: int) -> int:
    return -(-int(a) // int(b))


__all__ = [
    "WORKLOADS", "normal_f16", "layer_params", "activations", "decode_inputs",
    "kv_history", "codec_tensor", "codec_rows_for_bytes", "ceil_div", "math", "OPT_VOCAB", "model_params",
    "token_ids",
]
