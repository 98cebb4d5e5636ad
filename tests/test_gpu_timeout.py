"""Failure detection without a fault: the tensor-core GEMM's pipeline waits are bounded,
and flex_set_wait_limit_ns makes the bound short enough to run out on a wait of a few
microseconds. The kernel then records FLEX_ERR_TIMEOUT, stops, drains its own copies and
MMAs, frees its tensor memory and exits; flex_get_status reports the timeout and the
device stays usable: the same GEMM run right after with the default limit gives the
same bits as before. Nothing here breaks a kernel or faults the GPU: every wait in the
abort path keeps its own 2 s bound, and every thread still reaches every barrier.

Three launch forms of the split-K reduction are covered: no split (148 CTAs), splits
reduced through workspace tickets (96 tiles x 3 splits), and splits reduced inside a
thread-block cluster (1 tile x 8 splits)."""
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from _helpers import sync_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(144, 148 * 256, 1024),      # one 256-row tile per SM, no split
                                   (144, 96 * 256, 12288),      # 96 tiles x 3 splits, ticket reduction
                                   (144, 256, 49152)])          # 1 tile x 8 splits in one cluster
def test_short_wait_limit_times_out_then_next_call_is_exact(M, N, K):
    W = fq.CompressedWeight(synth.normal_f16((N, K), 40, 0.02, device="cuda"))
    x = synth.activations((M, K), 41, device="cuda")
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
    fq.flex_dequant_gemm(x, W, None, None, ref, M, fq.FLEX_EPI_NONE, ws)
    sync_status()
    old = fq.flex_set_wait_limit_ns(1)
    try:
        y = torch.zeros_like(ref)
        fq.flex_dequant_gemm(x, W, None, None, y, M, fq.FLEX_EPI_NONE, ws)
        rc = fq.flex_get_status()
    finally:
        fq.flex_set_wait_limit_ns(old)
    assert rc == fq.FLEX_ERR_TIMEOUT, fq.flex_status_string(rc)
    y = torch.zeros_like(ref)
    fq.flex_dequant_gemm(x, W, None, None, y, M, fq.FLEX_EPI_NONE, ws)
    sync_status()
    assert torch.equal(y, ref)
    assert not ws[:2048].any(), "split-K tickets must return to zero after an aborted call"
