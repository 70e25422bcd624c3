"""SwiGLU in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

The large-hidden DiT block's fused projection writes, next to the Q, K and V
features, 2 x d_ff gate and up features; the MLP's activation is
silu(gate) * up, the SwiGLU epilogue that the NVIDIA blog page on FLUX on
Blackwell fuses into the NVFP4 GEMM ("NVIDIA Technical Blog Details FLUX 3
Image Klein Blackwell Inference Optimization Methods", the NVFP4 / fused-GEMM
paragraph: SwiGLU, QKV projection and RoPE epilogues).  silu is the logistic
gate x * sigmoid(x) = x / (1 + exp(-x)).
"""
from __future__ import annotations

import numpy as np


def silu(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, np.float64)
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def swiglu(gate: np.ndarray, up: np.ndarray) -> np.ndarray:
    return silu(gate) * np.asarray(up, np.float64)


def split_fused(y: np.ndarray, n_plain: int, n_ff: int):
    """Outputs of a fused projection in its natural column order
    [plain (n_plain) | gate (n_ff) | up (n_ff)] -> (plain part, swiglu)."""
    y = np.asarray(y, np.float64)
    assert y.shape[1] == n_plain + 2 * n_ff
    return y[:, :n_plain], swiglu(y[:, n_plain:n_plain + n_ff], y[:, n_plain + n_ff:])
