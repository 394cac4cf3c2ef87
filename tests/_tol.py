"""Tolerance checks for the BCQ matmul against the FP64 oracle.

The bar for floating point: relative L2 error <= 1e-3 over the whole [batch][m]
output, and per output |y - y_ref| <= 2e-3 * A_j * ||x_b||_1 / n, where
A_j = sum_i mean_G |alpha[i, G, j]| (the per-row sum of plane scales; the mean
over groups is the stricter reading when alpha varies by group).
"""
from __future__ import annotations

import numpy as np

REL_L2 = 1e-3
ABS_COEF = 2e-3


def abs_bound(alpha, x, n: int) -> np.ndarray:
    """Per-output max-abs bound [batch][m]."""
    a = np.abs(np.asarray(alpha, dtype=np.float64))           # [q][ng][m]
    A = a.mean(axis=1).sum(axis=0)                           # [m]
    xl1 = np.abs(np.asarray(x, dtype=np.float64)).sum(axis=1)  # [batch]
    return ABS_COEF * A[None, :] * xl1[:, None] / float(n)


def compare(y, y_ref, alpha, x, n: int):
    """Returns (ok, stats) for y against y_ref under both criteria."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    assert y.shape == y_ref.shape, (y.shape, y_ref.shape)
    err = np.abs(y - y_ref)
    denom = np.linalg.norm(y_ref)
    rel = float(np.linalg.norm(y - y_ref) / denom) if denom > 0 else float(np.linalg.norm(y))
    bound = abs_bound(alpha, x, n)
    ratio = float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0
    finite = bool(np.all(np.isfinite(y)))
    ok = finite and rel <= REL_L2 and ratio <= 1.0
    return ok, {"rel_l2": rel, "max_abs_over_bound": ratio, "max_abs": float(err.max(initial=0.0)),
                "finite": finite}


def compare_f16(y16, y_ref, alpha, x, n: int):
    """fp16 output against the FP64 oracle: the fp16 mode is RNE of the fp32
    sum, so |y16 - y_ref| <= half an fp16 ulp (taken at the larger of |y16|,
    |y_ref|, which covers rounding up into the next binade) plus the fp32
    per-output bound.  Returns (ok, stats)."""
    y16 = np.asarray(y16, dtype=np.float16)
    y = y16.astype(np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    half_ulp = 0.5 * np.spacing(np.maximum(np.abs(y), np.abs(y_ref)).astype(np.float16)).astype(np.float64)
    bound = half_ulp + abs_bound(alpha, x, n)
    err = np.abs(y - y_ref)
    ratio = float((err / bound).max()) if err.size else 0.0
    finite = bool(np.all(np.isfinite(y)))
    return finite and ratio <= 1.0, {"max_err_over_bound": ratio, "finite": finite}
