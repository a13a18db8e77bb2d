"""Tolerances and tensor conversions shared by the GPU parity tests.

Bar (fp32 arithmetic inside every kernel, one rounding at each store):
  * bf16 outputs: |g - o| <= max(2 * ulp_bf16(o), 1e-3), ulp_bf16(o) = 2^(floor(log2|o|) - 7)
    (2 bf16 ulp with a 1e-3 absolute floor), and the relative error must stay below
    1.6e-2 wherever |o| > 1e-3;
  * fp32 outputs: |g - o| <= 1e-5 * |o| + 1e-6 (1e-5 relative; the 1e-6 floor covers
    results that cancel to ~0, where a relative bound alone is meaningless).
o is the fp64 oracle value, g the GPU value widened exactly to fp64.
"""
from __future__ import annotations

import numpy as np
import torch


def to_oracle(t: torch.Tensor | None) -> np.ndarray | None:
    """Device tensor -> contiguous host array of the same bits (bf16 as uint16)."""
    if t is None:
        return None
    c = t.detach().contiguous().cpu()
    if c.dtype == torch.bfloat16:
        return c.view(torch.int16).numpy().view(np.uint16).copy()
    if c.dtype == torch.float32:
        return c.numpy().copy()
    if c.dtype in (torch.int32, torch.uint8, torch.int64):
        return c.numpy().copy()
    raise TypeError(c.dtype)


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def tolerance(want: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    a = np.abs(want)
    if dtype == torch.bfloat16:
        with np.errstate(divide="ignore"):
            ulp = np.where(a > 0, np.exp2(np.floor(np.log2(np.where(a > 0, a, 1.0))) - 7), 0.0)
        return np.maximum(2.0 * ulp, 1e-3)
    return 1e-5 * a + 1e-6


def assert_close(got: np.ndarray, want: np.ndarray, dtype: torch.dtype, what: str = ""):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite GPU output"
    err = np.abs(got - want)
    tol = tolerance(want, dtype)
    bad = err > tol
    if bad.any():
        idx = np.unravel_index(np.argmax(err - tol), err.shape)
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; worst at {idx}: "
            f"gpu {got[idx]!r} oracle {want[idx]!r} err {err[idx]:.3e} tol {tol[idx]:.3e}")
    if dtype == torch.bfloat16:
        big = np.abs(want) > 1e-3
        if big.any():
            rel = (err[big] / np.abs(want[big])).max()
            assert rel <= 1.6e-2, f"{what}: max relative error {rel:.3e} > 1.6e-2"


def max_rel(got: np.ndarray, want: np.ndarray) -> float:
    big = np.abs(want) > 1e-3
    if not big.any():
        return 0.0
    return float((np.abs(got - want)[big] / np.abs(want[big])).max())
