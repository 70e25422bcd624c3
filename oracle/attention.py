"""FP8 attention in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

The NVIDIA blog page on FLUX on Blackwell quantises attention to FP8 as its
second optimisation layer ("NVIDIA Technical Blog Details FLUX 3 Image Klein
Blackwell Inference Optimization Methods", the paragraph after the NVFP4 /
fused-GEMM one: VC-Attention FP8 with a repair budget) without stating the
arithmetic.  The plainest reading, used here:

* queries, keys and values are each quantised to FP8 E4M3 with one fp32 scale
  per tensor, s = amax / 448 (1 when that is not a normal number), each
  element coded as E4M3_rn_satfinite(fl(x * fl(1/s))) -- the same steps as
  the NVFP4 block scales, with a signed code;
* attention itself is the exact scaled dot-product softmax of the
  dequantised tensors, per head h of d features:
      O[m, h] = sum_j softmax_j(c * <q_m, k_j>) v_j,   c = 1/sqrt(d).
  The GPU evaluates the same expression with fp32 scores, an online softmax
  and the probabilities rounded to E4M3 for the second product; the oracle
  is the exact value, and the tolerance covers that rounding.

The page's "repair" of the quantised attention is not defined there and is
not part of this reading.
"""
from __future__ import annotations

import numpy as np

from . import nvfp4

F32 = np.float32


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Signed fp32 -> E4M3 byte, round to nearest even, saturating at +-448;
    the sign bit is copied from the input (a negative value that rounds to
    zero gives 0x80)."""
    v = np.asarray(v, dtype=np.float32)
    mag = nvfp4.e4m3_encode_nonneg(np.abs(v))
    return (mag | (np.signbit(v).astype(np.uint8) << 7)).astype(np.uint8)


def fp8_scale(amax) -> np.float32:
    """Per-tensor scale amax / 448, or 1 when that is not a normal fp32 number."""
    s = F32(F32(amax) / F32(448.0))
    if not (s >= F32(1.17549435e-38)):
        s = F32(1.0)
    return s


def fp8_quantize(x: np.ndarray, amax=None):
    """x (bf16 values as fp32) -> (E4M3 codes, per-tensor scale s).  ``amax``
    gives the whole tensor's maximum magnitude when x is a part of it (every
    element is coded on its own once the scale is fixed)."""
    x = np.asarray(x, dtype=np.float32)
    if amax is None:
        amax = np.max(np.abs(x)) if x.size else F32(0.0)
    s = fp8_scale(amax)
    inv = F32(F32(1.0) / s)
    codes = e4m3_encode((x * inv).astype(np.float32))
    return codes, s


def fp8_dequantize(codes: np.ndarray, s) -> np.ndarray:
    return nvfp4.e4m3_decode(codes) * float(s)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, heads: int, scale=None) -> np.ndarray:
    """Exact softmax attention in fp64.  q, k, v [S, heads * d] token-major
    (head h in columns h*d .. h*d+d-1); returns O [S, heads * d]."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    d = q.shape[1] // heads
    c = 1.0 / np.sqrt(d) if scale is None else float(scale)
    out = np.empty((q.shape[0], v.shape[1]), np.float64)
    for h in range(heads):
        cols = slice(h * d, (h + 1) * d)
        s = c * (q[:, cols] @ k[:, cols].T)
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[:, cols] = (p @ v[:, cols]) / p.sum(axis=1, keepdims=True)
    return out
