"""Rotary position embedding in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

The NVIDIA blog page on FLUX on Blackwell lists RoPE beside SwiGLU and the
QKV projection as an epilogue fused into its NVFP4 GEMM ("NVIDIA Technical
Blog Details FLUX 3 Image Klein Blackwell Inference Optimization Methods",
the NVFP4 / fused-GEMM paragraph) and gives no formula.  The plainest reading
is the rotary embedding of Su et al. ("RoFormer: Enhanced Transformer with
Rotary Position Embedding", 2021, section 3.4): in every head of d features,
the feature pair (2i, 2i+1) of token m is turned by an angle theta[m, i],

    y'[2i]   = y[2i] cos theta - y[2i+1] sin theta
    y'[2i+1] = y[2i] sin theta + y[2i+1] cos theta,

the same angles for every head and for the query and key features.  RoFormer
takes theta[m, i] = m * base^(-2i/d); multi-axis variants (image tokens
with a row and a column position) give each axis its own run of pairs and its
own frequencies.  ``angles`` builds that schedule from integer positions;
``rotate`` takes any per-token, per-pair table, which is what the GPU epilogue
consumes (``table``: cos and sin interleaved, rounded once to fp32).
"""
from __future__ import annotations

import numpy as np


def angles(pos: np.ndarray, axes_dims, base: float) -> np.ndarray:
    """theta [M, d/2] for positions ``pos`` [M, n_axes] and per-axis feature
    counts ``axes_dims`` (even, summing to the head size d): axis a owns the
    next axes_dims[a] / 2 pairs, pair j of the axis turning at frequency
    base^(-2j / axes_dims[a]) per unit of that axis's position."""
    pos = np.asarray(pos, np.float64)
    if pos.ndim == 1:
        pos = pos[:, None]
    assert pos.shape[1] == len(axes_dims)
    cols = []
    for a, d_a in enumerate(axes_dims):
        assert d_a % 2 == 0
        freq = np.power(float(base), -np.arange(0, d_a, 2, dtype=np.float64) / d_a)
        cols.append(pos[:, a:a + 1] * freq[None, :])
    return np.concatenate(cols, axis=1)


def table(theta: np.ndarray) -> np.ndarray:
    """The epilogue's input: fp32 [M, d] with cos theta[m, i] at column 2i and
    sin theta[m, i] at column 2i + 1."""
    theta = np.asarray(theta, np.float64)
    t = np.empty((theta.shape[0], 2 * theta.shape[1]), np.float64)
    t[:, 0::2] = np.cos(theta)
    t[:, 1::2] = np.sin(theta)
    return t.astype(np.float32)


def rotate(y: np.ndarray, tab: np.ndarray, n_rope: int, d_head: int) -> np.ndarray:
    """y [M, N] (fp64) with its first n_rope columns, heads of d_head
    features, turned pair by pair by the table ``tab`` [M, >= d_head]
    (interleaved cos, sin as in ``table``); the other columns unchanged."""
    y = np.array(y, np.float64, copy=True)
    tab = np.asarray(tab, np.float64)
    assert n_rope % d_head == 0 and d_head % 2 == 0 and n_rope <= y.shape[1]
    c = tab[:, 0:d_head:2]
    s = tab[:, 1:d_head:2]
    for h0 in range(0, n_rope, d_head):
        even = y[:, h0:h0 + d_head:2].copy()
        odd = y[:, h0 + 1:h0 + d_head:2].copy()
        y[:, h0:h0 + d_head:2] = even * c - odd * s
        y[:, h0 + 1:h0 + d_head:2] = even * s + odd * c
    return y
