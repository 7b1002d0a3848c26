"""Shared helpers of the parity tests: the error metrics and device moves.

The metric follows the tolerance stated for the block: for bf16, the per-row
max-abs error normalised by the row's max-abs oracle value; for fp32, the same
per-row metric plus an element-wise relative error with a floor of 1e-3 of the
row maximum.
"""

import numpy as np
import torch

BF16_TOL = 2e-2   # per-row max-norm error vs the fp64 oracle
F32_TOL = 1e-4    # max relative error vs the fp64 oracle


def as_np(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def row_err(got, want) -> float:
    """max over rows of max_j |got - want| / max_j |want| (last axis = row)."""
    g, w = as_np(got), as_np(want)
    assert g.shape == w.shape, (g.shape, w.shape)
    g = g.reshape(-1, g.shape[-1])
    w = w.reshape(-1, w.shape[-1])
    assert np.all(np.isfinite(g)), "non-finite values in the GPU result"
    den = np.maximum(np.max(np.abs(w), axis=1), 1e-30)
    return float(np.max(np.max(np.abs(g - w), axis=1) / den))


def rel_err_floor(got, want, floor_frac=1e-3) -> float:
    """max element-wise |got - want| / max(|want|, floor_frac * rowmax |want|)."""
    g, w = as_np(got), as_np(want)
    g = g.reshape(-1, g.shape[-1])
    w = w.reshape(-1, w.shape[-1])
    floor = floor_frac * np.max(np.abs(w), axis=1, keepdims=True)
    return float(np.max(np.abs(g - w) / np.maximum(np.abs(w), np.maximum(floor, 1e-30))))


def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to("cuda")


def weights_to_cuda(w: dict) -> dict:
    return {k: cuda(v) for k, v in w.items()}
