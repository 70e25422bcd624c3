"""Dual-branch W4A4 forward pass in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

Follows "SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption":
pillar 1 ("Mathematical Outlier Factorization") gives the forward pass as the
4-bit GEMM of the quantised operands plus the low-rank branch evaluated right
to left, and section "Step 2: The SVDQuant Dual-Branch Linear Layer" adds the
bias after summing the two branches.  In the row-major token convention used
here (Y = X W^T, X [M, K], W [N, K]) that is

    Y = Q(X diag(s)^-1) Q(R)^T  +  (X L1) L2  +  bias

with L1 [K, r] (1/s folded in) and L2 [r, N].  The quantised product is the
exact fp64 product of the dequantised operands (a library matmul serves as
the contraction); the low-rank branch reads the raw bf16 X.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4


def lowrank_down(x_bf16_as_f32: np.ndarray, L1t: np.ndarray) -> np.ndarray:
    """U = X L1 in fp64; ``L1t`` is L1 transposed, [r, K]."""
    return np.asarray(x_bf16_as_f32, np.float64) @ np.asarray(L1t, np.float64).T


def w4a4_linear(x_bf16_as_f32, inv_s, Wq_packed, Wsf, t_w, L1t, L2t, bias=None,
                rows=None):
    """Reference output Y (fp64) of one W4A4 linear.

    x_bf16_as_f32 [M, K]  the activation's bf16 values as fp32
    inv_s         [K]     fp32 reciprocal smoothing factors (None = ones)
    Wq_packed     [N, K/2] packed E2M1 codes of the residual weight
    Wsf           [N, K/16] E4M3 block scales (row-major)
    t_w           fp32 per-tensor weight scale
    L1t [r, K], L2t [N, r]  low-rank factors (bf16 values as fp32), r may be 0
    bias [N] or None
    rows          optional row indices: evaluate only these rows of Y.  The
                  activation scale still comes from the whole tensor; only the
                  selected rows are quantised (rows are independent once the
                  tensor scale is fixed).
    The weight arguments may hold a subset of the output channels (with the
    matching L2t rows and bias entries); Y then has those columns only.
    Returns (Y fp64, dict of the activation quantisation results of the
    evaluated rows).
    """
    x = np.asarray(x_bf16_as_f32, np.float32)
    xq, xsf, t_x, amax = nvfp4.quantize_activation(x, inv_s, rows)
    sel = slice(None) if rows is None else np.asarray(rows)
    xdeq = nvfp4.dequantize(nvfp4.unpack(xq), xsf, t_x)
    wdeq = nvfp4.dequantize(nvfp4.unpack(Wq_packed), Wsf, t_w)
    y = xdeq @ wdeq.T
    if L1t is not None and np.asarray(L1t).shape[0] > 0:
        u = lowrank_down(x[sel], L1t)
        y = y + u @ np.asarray(L2t, np.float64).T
    if bias is not None:
        y = y + np.asarray(bias, np.float64)[None, :]
    return y, {"xq": xq, "xsf": xsf, "t_x": t_x, "amax": amax}


def rel_frobenius(y_test: np.ndarray, y_ref: np.ndarray) -> float:
    d = np.asarray(y_test, np.float64) - np.asarray(y_ref, np.float64)
    den = np.linalg.norm(np.asarray(y_ref, np.float64))
    return float(np.linalg.norm(d) / den) if den > 0 else float(np.linalg.norm(d))


def row_maxabs_ratio(y_test: np.ndarray, y_ref: np.ndarray) -> float:
    """max over rows of max|y_test - y_ref| / max|y_ref| (row-wise inf norms)."""
    d = np.abs(np.asarray(y_test, np.float64) - np.asarray(y_ref, np.float64)).max(axis=1)
    n = np.abs(np.asarray(y_ref, np.float64)).max(axis=1)
    n = np.where(n > 0, n, 1.0)
    return float((d / n).max()) if d.size else 0.0
