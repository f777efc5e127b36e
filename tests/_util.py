"""Shared helpers for the parity tests (no attention arithmetic here)."""

import numpy as np
import torch


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(got, ref) -> float:
    """max |got - ref| / max |ref| over all elements."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    return float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))


def abs_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    return float(np.max(np.abs(got - ref)))


# Parity bars (bf16 inputs, fp32 accumulation): max-abs error relative to the
# oracle's max-abs for O, dQ, dK, dV; absolute error for lse.
TOL_REL = 2e-2
TOL_LSE = 1e-3
