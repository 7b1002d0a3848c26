"""Shared helpers of the parity tests: the error metrics and device moves.

The metric follows the tolerance stated for the block: the per-row max-abs
error normalised by the row's max-abs oracle value (||got - want||_inf /
||want||_inf over the last axis), at most 2e-2 for bf16 and 1e-4 for fp32.
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


BF16_U = 2.0 ** -8  # unit roundoff of bf16 (8-bit significand, round to nearest)


def branch_err(y_got, y_want, x1_want, branch_want, u=BF16_U) -> float:
    """Error of the residual-free branch sum X'' - X, per row, normalised by the
    branch's max-abs value, after removing what the storage rounding of the
    residual stream itself allows: X' and X'' are each stored in the compute
    dtype, so element j may differ by up to u * (|X'_j| + |X''_j|) with an exact
    branch."""
    g, w = as_np(y_got), as_np(y_want)
    x1, br = as_np(x1_want), as_np(branch_want)
    g, w, x1, br = (a.reshape(-1, a.shape[-1]) for a in (g, w, x1, br))
    excess = np.maximum(np.abs(g - w) - u * (np.abs(x1) + np.abs(w)), 0.0)
    den = np.maximum(np.max(np.abs(br), axis=1), 1e-30)
    return float(np.max(np.max(excess, axis=1) / den))


def cuda(t: torch.Tensor) -> torch.Tensor:
    return t.contiguous().to("cuda")


def weights_to_cuda(w: dict) -> dict:
    return {k: cuda(v) for k, v in w.items()}
