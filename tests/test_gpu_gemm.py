"""Parity of the tcgen05 dequant-fused GEMM (flex_dequant_gemm, through the C ABI)
with the oracle: y = epilogue(x W^T + b) with W^ the oracle's dequantised weight,
float64 products. Tolerance: the method's max|err| <= 1e-2 max|ref| + 1e-3."""
import numpy as np
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from oracle import codec as oc
from _helpers import assert_layer_close, to_np, sync_status

pytestmark = pytest.mark.gpu


def _oracle_gemm(x, w16, bias, residual, epi, bits, rows=None):
    w = w16 if rows is None else w16[rows]
    c, m = oc.compress(np.ascontiguousarray(w), bits, 64, 1)
    wd = oc.decompress(c, m, w.shape, bits, 64, 1).astype(np.float64)
    y = x.astype(np.float64) @ wd.T
    if bias is not None:
        y += (bias if rows is None else bias[rows]).astype(np.float64)
    if epi == fq.FLEX_EPI_RELU:
        y = np.maximum(y, 0)
    if epi == fq.FLEX_EPI_RESIDUAL:
        y += (residual if rows is None else residual[:, rows]).astype(np.float64)
    return y


def _run(M, N, K, epi, bits=4, seed=0, with_bias=True):
    x = synth.activations((M, K), seed)
    w = synth.normal_f16((N, K), seed + 1, 0.02)
    b = synth.normal_f16((N,), seed + 2, 0.02) if with_bias else None
    r = synth.activations((M, N), seed + 3) if epi == fq.FLEX_EPI_RESIDUAL else None
    W = fq.CompressedWeight(w.cuda(), bits, 64)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    fq.flex_dequant_gemm(x.cuda(), W, None if b is None else b.cuda(), None if r is None else r.cuda(), y, M, epi, ws)
    sync_status()
    return x.numpy(), w.numpy(), None if b is None else b.numpy(), None if r is None else r.numpy(), y, ws


CASES = [(1, 256, 256), (4, 256, 512), (17, 384, 768), (32, 512, 2048), (48, 256, 256), (64, 768, 512),
         (144, 512, 1024), (250, 256, 512), (256, 384, 256), (300, 256, 512), (1000, 384, 768)]


@pytest.mark.parametrize("M,N,K", CASES)
def test_gemm_bias(M, N, K):
    x, w, b, _, y, _ = _run(M, N, K, fq.FLEX_EPI_NONE, seed=M)
    assert_layer_close(y, _oracle_gemm(x, w, b, None, fq.FLEX_EPI_NONE, 4), f"gemm {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(4, 256, 512), (144, 512, 1024), (700, 256, 256)])
def test_gemm_relu(M, N, K):
    x, w, b, _, y, _ = _run(M, N, K, fq.FLEX_EPI_RELU, seed=M + 7)
    ref = _oracle_gemm(x, w, b, None, fq.FLEX_EPI_RELU, 4)
    assert_layer_close(y, ref, "relu")
    assert float(y.min()) >= 0


@pytest.mark.parametrize("M,N,K", [(5, 256, 768), (144, 384, 512), (513, 256, 256)])
def test_gemm_residual(M, N, K):
    x, w, b, r, y, _ = _run(M, N, K, fq.FLEX_EPI_RESIDUAL, seed=M + 9)
    assert_layer_close(y, _oracle_gemm(x, w, b, r, fq.FLEX_EPI_RESIDUAL, 4), "residual")


@pytest.mark.parametrize("M,N,K", [(8, 256, 512), (200, 256, 768)])
def test_gemm_8bit_no_bias(M, N, K):
    x, w, _, _, y, _ = _run(M, N, K, fq.FLEX_EPI_NONE, bits=8, seed=M + 11, with_bias=False)
    assert_layer_close(y, _oracle_gemm(x, w, None, None, fq.FLEX_EPI_NONE, 8), "8-bit")


@pytest.mark.parametrize("M,N,K", [(32, 19200, 4096), (512, 9472, 2048), (144, 19200, 2048)])
def test_gemm_ring_reuse(M, N, K):
    """Enough tiles for a single K split, so every shared-memory ring wraps around
    several times (the code/metadata stages, the activation and the dequantised rings)."""
    x = synth.activations((M, K), 60, device="cuda")
    w = synth.normal_f16((N, K), 61, 0.02, device="cuda")
    b = synth.normal_f16((N,), 62, 0.02, device="cuda")
    W = fq.CompressedWeight(w, 4, 64)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    fq.flex_dequant_gemm(x, W, b, None, y, M, 0, ws)
    sync_status()
    rows = np.array([0, 1, 127, 128, 5000 % N, N - 129, N - 1])
    mrows = np.unique(np.array([0, M // 2, M - 1]))
    ref = _oracle_gemm(to_np(x[torch.from_numpy(mrows).cuda()]), to_np(w), to_np(b), None, 0, 4, rows=rows)
    got = y[torch.from_numpy(mrows).cuda()][:, torch.from_numpy(rows).cuda()]
    assert_layer_close(got, ref, f"ring reuse {M}x{N}x{K}")


@pytest.mark.parametrize("M", [4, 16, 48])
def test_gemm_split_k_repeatable(M):
    """Split-K reduces in split order (M = 4, 16: the small-batch GEMV; M = 48: the
    tensor-core GEMM): two calls give identical bits, and a workspace, where one is
    needed, has its tickets back at zero after each call."""
    N, K = 512, 4096
    x, w, b, _, y1, ws = _run(M, N, K, fq.FLEX_EPI_NONE, seed=5)
    W = fq.CompressedWeight(torch.from_numpy(w).cuda(), 4, 64)
    y2 = torch.empty_like(y1)
    need = fq.flex_gemm_ws_bytes(M, N, K)
    fq.flex_dequant_gemm(torch.from_numpy(x).cuda(), W, torch.from_numpy(b).cuda(), None, y2, M, 0,
                         ws if need > 0 else None)
    sync_status()
    assert torch.equal(y1, y2)
    if need > 0:
        assert int(ws[:256].view(torch.int32).abs().sum()) == 0


@pytest.mark.parametrize("M,N,K", [(8, 128, 8192), (32, 128, 16384), (3, 256, 8192)])
def test_gemv_many_splits(M, N, K):
    """A narrow, deep GEMV splits K more ways than one cluster holds (16 or 32 splits),
    so its partials go through the workspace and the ticket: parity with the oracle,
    identical bits on a second call, tickets back at zero."""
    x, w, b, _, y1, ws = _run(M, N, K, fq.FLEX_EPI_NONE, seed=K + M)
    need = fq.flex_gemm_ws_bytes(M, N, K)
    assert need > 0
    assert_layer_close(y1, _oracle_gemm(x, w, b, None, fq.FLEX_EPI_NONE, 4), f"gemv {M}x{N}x{K}")
    W = fq.CompressedWeight(torch.from_numpy(w).cuda(), 4, 64)
    y2 = torch.empty_like(y1)
    fq.flex_dequant_gemm(torch.from_numpy(x).cuda(), W, torch.from_numpy(b).cuda(), None, y2, M, 0, ws)
    sync_status()
    assert torch.equal(y1, y2)
    assert int(ws[:256].view(torch.int32).abs().sum()) == 0


@pytest.mark.parametrize("name,M,N,K", [("opt-1.3b qkv decode", 32, 6144, 2048),
                                        ("opt-1.3b fc2 decode", 32, 2048, 8192),
                                        ("opt-30b fc1 gpu-batch", 48, 28672, 7168),
                                        ("opt-175b fc1 decode", 144, 49152, 12288),
                                        ("opt-1.3b qkv prefill", 16384, 6144, 2048)])
def test_gemm_full_size_sampled(name, M, N, K):
    """Full-size shapes in the launch configuration the layer uses; the oracle checks
    sampled output features (all tokens) - it needs only those weight rows."""
    x = synth.activations((M, K), 40, device="cuda")
    w = synth.normal_f16((N, K), 41, 0.02, device="cuda")
    b = synth.normal_f16((N,), 42, 0.02, device="cuda")
    W = fq.CompressedWeight(w, 4, 64)
    y = torch.empty((M, N), dtype=torch.float16, device="cuda")
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    fq.flex_dequant_gemm(x, W, b, None, y, M, 0, ws)
    sync_status()
    rng = np.random.default_rng(N)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 1], rng.integers(0, N, 24)]))
    mrows = np.unique(np.concatenate([[0, M - 1], rng.integers(0, M, 64)])) if M > 256 else np.arange(M)
    xs = to_np(x[torch.from_numpy(mrows).cuda()])
    ref = _oracle_gemm(xs, to_np(w), to_np(b), None, 0, 4, rows=rows)
    got = y[torch.from_numpy(mrows).cuda()][:, torch.from_numpy(rows).cuda()]
    assert_layer_close(got, ref, name)
    assert bool(torch.isfinite(y).all())


def test_gemm_bad_args():
    w = torch.zeros((256, 512), dtype=torch.float16, device="cuda")
    W = fq.CompressedWeight(w)
    y = torch.empty((4, 256), dtype=torch.float16, device="cuda")
    x = torch.zeros((4, 512), dtype=torch.float16, device="cuda")
    # a narrow, deep shape split along K into more parts than one cluster holds needs
    # the workspace reduction: a missing workspace is refused before launch
    assert fq.flex_gemm_ws_bytes(8, 128, 8192) > 0
    W2 = fq.CompressedWeight(torch.zeros((128, 8192), dtype=torch.float16, device="cuda"))
    x2 = torch.zeros((8, 8192), dtype=torch.float16, device="cuda")
    y2 = torch.empty((8, 128), dtype=torch.float16, device="cuda")
    with pytest.raises(fq.FlexError) as e:
        fq.flex_dequant_gemm(x2, W2, None, None, y2, 8, fq.FLEX_EPI_NONE, None)
    assert e.value.code == fq.FLEX_ERR_WORKSPACE
    with pytest.raises(fq.FlexError) as e:
        fq.flex_dequant_gemm(x, W, None, None, y, 4, fq.FLEX_EPI_RESIDUAL, None)
    assert e.value.code == fq.FLEX_ERR_INVALID_ARG


def test_gemm_sequence_shares_one_workspace():
    """GEMMs of different tile counts and split counts run back to back on one
    workspace, as inside a layer call: every result matches its own run on a fresh
    workspace (a GEMM's partials must never land on another's tickets)."""
    shapes = [(32, 6144, 2048), (32, 2048, 2048), (32, 8192, 2048), (32, 2048, 8192), (48, 2048, 2048),
              (48, 6144, 2048)]
    need = max(fq.flex_gemm_ws_bytes(*s) for s in shapes)
    shared = torch.zeros(max(16, need), dtype=torch.uint8, device="cuda")
    for rep in range(2):
        for i, (M, N, K) in enumerate(shapes):
            x = synth.activations((M, K), 60 + i, device="cuda")
            W = fq.CompressedWeight(synth.normal_f16((N, K), 70 + i, 0.02, device="cuda"))
            y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
            y2 = torch.empty_like(y1)
            fq.flex_dequant_gemm(x, W, None, None, y1, M, 0, shared)
            fresh = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
            fq.flex_dequant_gemm(x, W, None, None, y2, M, 0, fresh)
            sync_status()
            assert torch.equal(y1, y2), (rep, M, N, K)


def _interleave8(x):
    """Every 8-block of the last dim as [k0, k4, k1, k5, k2, k6, k3, k7]."""
    s = x.shape
    b = x.reshape(*s[:-1], s[-1] // 8, 2, 4).transpose(-1, -2)
    return b.reshape(s).contiguous()


@pytest.mark.parametrize("M,N,K", [(32, 2048, 2048), (7, 512, 1024), (48, 1024, 2048)])
def test_gemm_interleaved_activations(M, N, K):
    """FLEX_GEMM_X_INTERLEAVED: the same logical activations stored in the interleaved
    8-block order give the natural-order result (bit for bit on the small-batch path,
    whose operands are identical; within rounding on the tensor-core GEMM, whose K order
    changes)."""
    x = synth.activations((M, K), 80, device="cuda")
    W = fq.CompressedWeight(synth.normal_f16((N, K), 81, 0.02, device="cuda"))
    y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
    y2 = torch.empty_like(y1)
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    fq.flex_dequant_gemm(x, W, None, None, y1, M, fq.FLEX_EPI_NONE, ws)
    fq.flex_dequant_gemm(_interleave8(x), W, None, None, y2, M, fq.FLEX_EPI_NONE | fq.FLEX_GEMM_X_INTERLEAVED, ws)
    sync_status()
    if M <= 32:
        assert torch.equal(y1, y2)
    else:
        assert (y1.float() - y2.float()).abs().max().item() <= 1e-2 * y1.float().abs().max().item() + 1e-3


def _plan_cases():
    """(M, N, K) candidates whose plans cover the split-K reduction paths of the two
    tensor-core kernels: no split, splits through a thread-block cluster, through the
    workspace ticket with at most 4 and with more than 4 splits, and stream-K."""
    cands = []
    for M in (48, 144):
        for tiles in (1, 2, 6, 12, 20, 24, 28, 40, 96, 192):
            for K in (2048, 12288, 49152):
                N = tiles * (256 if M > 128 else 128)
                cands.append((M, N, K))
    return cands


def _path(pl):
    if pl["reduce"] in ("none", "cluster", "streamk", "exchange"):
        return (pl["kernel"], pl["reduce"])
    return (pl["kernel"], "ticket<=4" if pl["splits"] <= 4 else "ticket>4")


@pytest.mark.parametrize("streamk", [True, False])
def test_gemm_split_reduction_paths(streamk):
    """Every split-K reduction path the device's plans reach is parity-checked against
    the oracle on sampled output features and gives identical bits on a second call;
    the workspace tickets and stream-K flags are back at zero. Required: both ticket
    paths (at most 4 splits, and more: the partials are added 4 at a time) of the
    128-row kernel; stream-K and the one-wave exchange of the 256-row kernel (and its
    ticket path wherever the candidates reach it)."""
    old = fq.flex_set_gemm_streamk(streamk)
    try:
        seen = {}
        for M, N, K in _plan_cases():
            path = _path(fq.flex_gemm_plan(M, N, K))
            if path not in seen or N * K < seen[path][1] * seen[path][2]:
                seen[path] = (M, N, K)
        need = [("tc128", "ticket<=4"), ("tc128", "ticket>4")]
        need += ([("tc256", "streamk"), ("tc256", "exchange")] if streamk
                 else [("tc256", "exchange"), ("tc256", "ticket<=4")])
        for k in need:
            assert k in seen, sorted(seen)
        for path, (M, N, K) in sorted(seen.items()):
            x = synth.activations((M, K), 90, device="cuda")
            w = synth.normal_f16((N, K), 91, 0.02, device="cuda")
            W = fq.CompressedWeight(w, 4, 64)
            ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
            y1 = torch.empty((M, N), dtype=torch.float16, device="cuda")
            y2 = torch.empty_like(y1)
            fq.flex_dequant_gemm(x, W, None, None, y1, M, fq.FLEX_EPI_NONE, ws)
            fq.flex_dequant_gemm(x, W, None, None, y2, M, fq.FLEX_EPI_NONE, ws)
            sync_status()
            assert torch.equal(y1, y2), path
            assert int(ws[:2048].view(torch.int32).abs().sum()) == 0, path
            rows = np.unique(np.linspace(0, N - 1, 24).astype(np.int64))
            ref = _oracle_gemm(to_np(x), to_np(w), None, None, fq.FLEX_EPI_NONE, 4, rows=rows)
            assert_layer_close(y1[:, torch.from_numpy(rows).cuda()], ref, f"{path} {M}x{N}x{K}")
            # every tile of the whole output is finished: full-row check of a few tokens
            mrows = [0, M // 2, M - 1]
            wd = fq.flexq_decompress(W.codes, W.meta, W.shape, W.cfg).float()
            full = x[mrows].float() @ wd.t()
            err = (y1[mrows].float() - full).abs().max().item()
            assert err <= 1e-2 * full.abs().max().item() + 1e-3, (path, err)
    finally:
        fq.flex_set_gemm_streamk(old)


@pytest.mark.parametrize("M,N,K", [(4, 256, 512), (32, 512, 2048)])
def test_small_batches_on_the_tensor_core_gemm(M, N, K):
    """flex_set_gemm_gemv(False) sends batches of up to 32 rows to the 128-row tcgen05
    GEMM (the comparison the route switch exists for); it must give the same result
    within the tolerance, and the default route comes back afterwards."""
    assert fq.flex_gemm_plan(M, N, K)["kernel"] == "gemv"
    old = fq.flex_set_gemm_gemv(False)
    try:
        assert fq.flex_gemm_plan(M, N, K)["kernel"] == "tc128"
        x, w, b, _, y, _ = _run(M, N, K, fq.FLEX_EPI_NONE, seed=M + 31)
    finally:
        fq.flex_set_gemm_gemv(old)
    assert fq.flex_gemm_plan(M, N, K)["kernel"] == "gemv"
    assert_layer_close(y, _oracle_gemm(x, w, b, None, fq.FLEX_EPI_NONE, 4), f"tc128 {M}x{N}x{K}")
