"""Shared test helpers: numpy <-> torch for stored activations, and the
parity criteria used throughout the GPU tests.

Tolerances (float outputs compared with the float64 oracle run on the same
stored inputs):
  float32 activations: |gpu - ref| <= 1e-4 * (1 + |ref|) element-wise.
  float32 backward pass ("f32bwd"): |gpu - ref| <= 1e-3 (|ref| + rms(ref)):
    the derivatives run two more recurrences (the recomputed states and the
    adjoint) and the sums over channels and time add up to 2^16 float32 terms.
  bfloat16 activations: |gpu - ref| <= 2e-2 * |ref| + 1e-3 * rms(ref)
    element-wise (2% relative, with an absolute floor of 0.1% of the tensor's
    RMS for values that cancel to near zero), and ||gpu - ref||_2 / ||ref||_2
    <= 5e-3.  The final state h_last is compared the same way.
"""
from __future__ import annotations

import numpy as np
import torch


def to_dev(a, device="cuda"):
    """numpy array (float32, or uint16 bf16 bits) -> torch tensor on device."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(a).to(device)


def to_np64(t):
    """torch tensor (bf16 or f32, any device) -> float64 numpy."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(got, ref, dtype, what=""):
    """Assert the parity criterion for `dtype` ("f32" or "bf16"); return stats."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite GPU values"
    err = np.abs(got - ref)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    if dtype == "f32":
        lim = 1e-4 * (1.0 + np.abs(ref))
    elif dtype == "f32bwd":
        lim = 1e-3 * (np.abs(ref) + rms)
    else:
        lim = 2e-2 * np.abs(ref) + 1e-3 * rms
    bad = err > lim
    nl2 = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300))
    stats = dict(max_abs=float(err.max()) if err.size else 0.0, nl2=nl2, rms=rms,
                 worst_ratio=float((err / lim).max()) if err.size else 0.0)
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(f"{what}: {int(bad.sum())} elements out of tolerance; first at {i}: "
                             f"gpu={got[i]!r} ref={ref[i]!r}; {stats}")
    if dtype not in ("f32", "f32bwd"):
        assert nl2 <= 5e-3, f"{what}: normalised L2 error {nl2:.3e} > 5e-3; {stats}"
    return stats
