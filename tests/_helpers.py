"""Shared helpers of the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch

import group_wise_int4_b200 as fq


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def u8(t) -> np.ndarray:
    return to_np(t).astype(np.uint8)


def assert_bits_equal(gpu: torch.Tensor, ref: np.ndarray, what: str):
    """Bit-exact comparison (fp16 compared through their uint16 patterns)."""
    g = to_np(gpu)
    if g.dtype == np.float16:
        g = g.view(np.uint16)
        ref = np.ascontiguousarray(ref).view(np.uint16)
    assert g.shape == ref.shape, (what, g.shape, ref.shape)
    bad = np.argwhere(g != ref)
    assert bad.size == 0, f"{what}: {len(bad)} mismatches, first at {bad[:5].tolist()}"


def layer_tolerance(ref: np.ndarray) -> float:
    """Layer-output tolerance of the method: max|err| <= 1e-2 * max|ref| + 1e-3."""
    return 1e-2 * float(np.max(np.abs(ref.astype(np.float64)))) + 1e-3


def assert_layer_close(gpu: torch.Tensor, ref: np.ndarray, what: str):
    g = to_np(gpu).astype(np.float64)
    r = ref.astype(np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    assert np.all(np.isfinite(g)), what
    err = float(np.max(np.abs(g - r))) if g.size else 0.0
    tol = layer_tolerance(r) if r.size else 0.0
    assert err <= tol, f"{what}: max|err| {err:.3e} > tol {tol:.3e}"
    return err, tol


def device():
    return torch.device("cuda:0")


def sync_status():
    rc = fq.flex_get_status()
    assert rc == fq.FLEX_OK, fq.flex_status_string(rc)
