"""NVFP4 formats and tensor quantiser -- oracle (TEST INFRASTRUCTURE ONLY).

Only tests, the smoke check and the CPU-baseline legs of the benchmark use this
module; the product path never does.

Sources
-------
* NVFP4 is the 4-bit format that the pages name for FLUX inference on
  Blackwell ("NVIDIA Technical Blog Details FLUX 3 Image Klein Blackwell
  Inference Optimization Methods ...", first optimisation layer; and the
  "FLUX.2 [klein] 4B base" model card, quantisation tip).  The pages never
  spell out its bit layout, so the layout used here is the one the library
  documents: E2M1 element codes {0, +-0.5, +-1, +-1.5, +-2, +-3, +-4, +-6},
  one unsigned E4M3 scale per 16 consecutive elements along K, one FP32 scale
  per tensor.
* E4M3's finite range of +-448 is quoted on "Quantization for the impatient --
  why int4 doesn't speed up image generation on GPU", section "Stability
  table".

Readings taken where the pages are silent (each one is listed in the design
notes):
1. Per-tensor scale ``t = A / (6 * 448)`` with ``A`` the tensor's absolute
   maximum, so the largest block lands on the largest E4M3 scale.  If ``t`` is
   not a normal fp32 number (``A == 0`` or tiny), ``t = 1``.
2. Block scale ``e = E4M3_rne_sat((b * (1/t)) / 6)`` with ``b`` the block's
   absolute maximum; every operation is one correctly-rounded fp32 operation,
   in that order.
3. Element code ``q = E2M1_rne_sat(x * (1 / (dec(e) * t)))``, again one fp32
   operation at a time.  A block whose scale decodes to zero gets all codes
   +0.  A negative value that rounds to zero keeps its sign (code 0x8).
4. Two codes per byte, the element with the even K index in the low nibble.

Rounding decisions are taken in IEEE fp32 (numpy float32 arithmetic is
correctly rounded, one operation at a time, no contraction); decoding and
everything downstream is exact in fp64.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32

# --------------------------------------------------------------------------
# E2M1: 1 sign bit (bit 3), 2 exponent bits (bias 1), 1 mantissa bit.
# --------------------------------------------------------------------------


def e2m1_decode_code(code: int) -> float:
    """Value of one 4-bit E2M1 code, from the bit fields."""
    sign = -1.0 if (code >> 3) & 1 else 1.0
    exp = (code >> 1) & 3
    man = code & 1
    if exp == 0:                      # subnormal: 0.m * 2^(1-bias) = m * 0.5
        mag = man * 0.5
    else:                             # normal: 1.m * 2^(exp-bias)
        mag = (1.0 + 0.5 * man) * 2.0 ** (exp - 1)
    return sign * mag


E2M1_VALUES = np.array([e2m1_decode_code(c) for c in range(16)], dtype=np.float64)
# magnitudes of the 8 non-negative codes, increasing with the code
E2M1_MAGS = E2M1_VALUES[:8].copy()


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    return E2M1_VALUES[np.asarray(codes, dtype=np.int64) & 15]


def _rne_onto_grid(a: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index of the grid point nearest to each non-negative ``a``.

    ``grid`` is increasing; the index doubles as the code, whose lowest bit is
    the mantissa LSB, so "ties to even" means "ties to the even index".
    Values at or beyond the last grid point saturate to it.  Distances are
    exact in fp64 because every operand is an fp32 value.
    """
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(grid, a, side="left")          # grid[hi-1] < a <= grid[hi]
    hi = np.clip(hi, 1, len(grid) - 1)
    lo = hi - 1
    d_lo = a - grid[lo]
    d_hi = grid[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(a >= grid[-1], len(grid) - 1, idx)  # satfinite
    idx = np.where(a <= 0.0, 0, idx)
    return idx.astype(np.int64)


def e2m1_encode(v: np.ndarray) -> np.ndarray:
    """fp32 -> E2M1 code, round to nearest even, saturating at +-6.

    The sign bit is copied from the input, so negative values (and -0.0)
    that round to zero give code 0x8.
    """
    v = np.asarray(v, dtype=np.float32)
    idx = _rne_onto_grid(np.abs(v).astype(np.float64), E2M1_MAGS)
    return (idx | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


# --------------------------------------------------------------------------
# E4M3 ("fn" variant): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits,
# no infinities, 0x7F / 0xFF are NaN, largest finite 0x7E = 448.
# --------------------------------------------------------------------------


def e4m3_decode_byte(b: int) -> float:
    sign = -1.0 if (b >> 7) & 1 else 1.0
    exp = (b >> 3) & 15
    man = b & 7
    if exp == 15 and man == 7:
        return float("nan")
    if exp == 0:                      # subnormal: 0.mmm * 2^(1-7)
        mag = (man / 8.0) * 2.0 ** -6
    else:
        mag = (1.0 + man / 8.0) * 2.0 ** (exp - 7)
    return sign * mag


E4M3_VALUES = np.array([e4m3_decode_byte(b) for b in range(256)], dtype=np.float64)
# magnitudes of the 127 non-negative finite codes 0x00..0x7E, increasing
E4M3_MAGS = E4M3_VALUES[:127].copy()
E4M3_MAX = 448.0


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    return E4M3_VALUES[np.asarray(b, dtype=np.int64) & 255]


def e4m3_encode_nonneg(v: np.ndarray) -> np.ndarray:
    """Non-negative fp32 -> E4M3 byte, round to nearest even, saturating at 448."""
    v = np.asarray(v, dtype=np.float32)
    if np.any(v < 0) or np.any(~np.isfinite(v)):
        raise ValueError("block scales are finite and non-negative")
    return _rne_onto_grid(v.astype(np.float64), E4M3_MAGS).astype(np.uint8)


# --------------------------------------------------------------------------
# Tensor quantiser
# --------------------------------------------------------------------------

BLOCK = 16
TENSOR_SCALE_DIVISOR = F32(6.0 * 448.0)      # 2688: E2M1 max times E4M3 max


def smooth(x_bf16_as_f32: np.ndarray, inv_s: np.ndarray | None) -> np.ndarray:
    """x~ = fl32(x * inv_s) per column (channel).

    Channel smoothing moves activation range into the weight, X' = X diag(s)^-1
    ("SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption", pillar 2,
    "SmoothQuant Pre-Conditioning for DiTs").
    """
    x = np.asarray(x_bf16_as_f32, dtype=np.float32)
    if inv_s is None:
        return x.copy()
    return (x * np.asarray(inv_s, dtype=np.float32)[None, :]).astype(np.float32)


def tensor_scale(amax: np.float32) -> np.float32:
    """Per-tensor FP32 scale t = A / 2688 (reading 1), t = 1 when not normal."""
    t = F32(F32(amax) / TENSOR_SCALE_DIVISOR)
    if not (t >= F32(2.0 ** -126)):
        t = F32(1.0)
    return t


def quantize(xs: np.ndarray, amax=None, t=None):
    """Quantise an already-smoothed fp32 matrix [rows, K] to NVFP4.

    ``amax`` is the tensor's absolute maximum; when the rows given are a
    subset of a larger tensor, pass the whole tensor's maximum (once the
    tensor scale is fixed, every row is quantised independently of the
    others).  ``t``, if given, is the tensor scale itself (a static or
    previous-step scale, the calibrated alternative that "SVDQuant Guide:
    4-Bit DiT Acceleration & Outlier Absorption", "1. Timestep-Aware Outlier
    Calibration" describes) and replaces ``tensor_scale(amax)``; the block
    scales and codes follow from it by the same steps, saturating where the
    data exceed what it can express.  Returns ``(codes u8 [rows, K],
    sf u8 [rows, K/16], t f32, amax f32)``; codes are unpacked (one per byte,
    see ``pack``).
    """
    xs = np.asarray(xs, dtype=np.float32)
    rows, K = xs.shape
    if K % BLOCK:
        raise ValueError("K must be a multiple of 16")
    if amax is None:
        amax = F32(np.max(np.abs(xs))) if xs.size else F32(0.0)
    amax = F32(amax)
    if t is None:
        t = tensor_scale(amax)
    else:
        t = F32(t)
        if not (t >= F32(2.0 ** -126)) or not np.isfinite(t):
            raise ValueError("a given tensor scale must be a normal positive fp32 number")
    rt = F32(F32(1.0) / t)
    blocks = xs.reshape(rows, K // BLOCK, BLOCK)
    bmax = np.max(np.abs(blocks), axis=2).astype(np.float32)          # b
    p = (bmax * rt).astype(np.float32)                                  # b * (1/t)
    s_raw = (p / F32(6.0)).astype(np.float32)                           # / 6
    sf = e4m3_encode_nonneg(s_raw)                                      # E4M3 byte
    sd = e4m3_decode(sf).astype(np.float32)                             # exact
    qscale = (sd * t).astype(np.float32)                                # dec(e) * t
    with np.errstate(divide="ignore"):
        rq = np.where(sd > 0, F32(1.0) / np.where(sd > 0, qscale, F32(1.0)), F32(0.0)).astype(np.float32)
    v = (blocks * rq[:, :, None]).astype(np.float32)                    # x * (1/(dec(e) t))
    codes = e2m1_encode(v)
    codes = np.where((sd > 0)[:, :, None], codes, np.uint8(0)).astype(np.uint8)
    return codes.reshape(rows, K), sf, t, amax


def pack(codes: np.ndarray) -> np.ndarray:
    """Two codes per byte: element 2i in the low nibble, 2i+1 in the high."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 15
    out[..., 1::2] = p >> 4
    return out


def dequantize(codes: np.ndarray, sf: np.ndarray, t) -> np.ndarray:
    """fp64 value of each element: dec(code) * dec(scale) * t (exact)."""
    rows, K = codes.shape
    v = e2m1_decode(codes).reshape(rows, K // BLOCK, BLOCK)
    v = v * e4m3_decode(sf)[:, :, None] * float(t)
    return v.reshape(rows, K)


def quantize_activation(x_bf16_as_f32: np.ndarray, inv_s: np.ndarray | None, rows=None):
    """Smooth, then quantise.  Returns (packed codes, sf, t, amax).

    With ``rows`` (indices), only those rows are quantised, under the tensor
    scale of the whole matrix.
    """
    xs = smooth(x_bf16_as_f32, inv_s)
    if rows is None:
        codes, sf, t, amax = quantize(xs)
    else:
        amax = F32(np.max(np.abs(xs))) if xs.size else F32(0.0)
        codes, sf, t, amax = quantize(xs[np.asarray(rows)], amax=amax)
    return pack(codes), sf, t, amax
