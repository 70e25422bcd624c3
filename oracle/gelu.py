"""tanh-approximated GELU in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

The single-stream DiT MLP applies GELU (tanh form) between its up- and
down-projections; the formula is the standard one,
0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))).
"""
from __future__ import annotations

import numpy as np


def gelu_tanh(x: np.ndarray) -> np.ndarray:
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (x + 0.044715 * x ** 3)))
