"""Failure detection without a fault: the tensor-core GEMM's waits are bounded, and a
test can make one run out with a flag that nothing sets.

flex_set_gemm_gate hands every later GEMM launch a device flag that its weight loader
waits on before the first load; the test passes a zero that nothing changes and a short
wait limit (flex_set_wait_limit_ns). The loader's wait then runs out: the kernel records
FLEX_ERR_TIMEOUT, every role sees the abort, the copies and MMAs already issued drain,
tensor memory is freed and the kernel exits. flex_get_status reports the timeout and
the device stays usable: the same GEMM run right after, without the gate and with the
default limit, gives the same bits as before. Nothing here breaks a kernel or faults the
GPU: every wait keeps a limit, and every thread still reaches every barrier.

(An earlier form of this test set the limit to 1 ns on the real pipeline waits. It saw
no timeout: an mbarrier try_wait may suspend until the phase completes, so waits that
complete within one poll never run out.)

Covered: the 256-row kernel with no split (148 CTAs), with the stream-K schedule (96
tiles of 3 splits' worth of work), with splits exchanging partials in one wave (48 tiles
x 3 splits) and with splits reduced inside a thread-block cluster (1 tile x 8 splits);
the 128-row kernel (N not a multiple of 256) with and without a split. (A wait that
gives up in the exchange or in stream-K still publishes this CTA's flag, so no peer
waits for it past its own limit.)"""
import pytest
import torch

import group_wise_int4_b200 as fq
import synth
from _helpers import sync_status

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K", [(144, 148 * 256, 1024),      # 256-row tiles, one per SM, no split
                                   (144, 96 * 256, 12288),      # 96 tiles x 3 splits in 2 waves: stream-K
                                   (144, 48 * 256, 12288),      # 48 x 3 splits in one wave: exchange
                                   (144, 256, 49152),           # 1 tile x 8 splits in one cluster
                                   (144, 37 * 128, 1024),       # 128-row kernel
                                   (144, 128, 49152)])          # 128-row kernel, 1 tile x 8 splits
def test_gated_loader_times_out_then_next_call_is_exact(M, N, K):
    W = fq.CompressedWeight(synth.normal_f16((N, K), 40, 0.02, device="cuda"))
    x = synth.activations((M, K), 41, device="cuda")
    ws = torch.zeros(max(16, fq.flex_gemm_ws_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
    ref = torch.empty((M, N), dtype=torch.float16, device="cuda")
    fq.flex_dequant_gemm(x, W, None, None, ref, M, fq.FLEX_EPI_NONE, ws)
    sync_status()
    gate = torch.zeros(1, dtype=torch.int32, device="cuda")      # nothing ever sets it
    old_limit = fq.flex_set_wait_limit_ns(5_000_000)             # 5 ms
    fq.flex_set_gemm_gate(gate)
    try:
        y = torch.zeros_like(ref)
        fq.flex_dequant_gemm(x, W, None, None, y, M, fq.FLEX_EPI_NONE, ws)
        rc = fq.flex_get_status()
    finally:
        fq.flex_set_gemm_gate(None)
        fq.flex_set_wait_limit_ns(old_limit)
    assert rc == fq.FLEX_ERR_TIMEOUT, fq.flex_status_string(rc)
    assert fq.flex_get_status() == fq.FLEX_OK                    # the status word was cleared
    y = torch.zeros_like(ref)
    fq.flex_dequant_gemm(x, W, None, None, y, M, fq.FLEX_EPI_NONE, ws)
    sync_status()
    assert torch.equal(y, ref)
    assert not ws[:2048].any(), "split-K tickets must return to zero after an aborted call"
