"""Offline SVDQuant preparation in fp64 -- oracle (TEST INFRASTRUCTURE ONLY).

"SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption":
* pillar 2 ("SmoothQuant Pre-Conditioning for DiTs"): W' = W diag(s),
  X' = diag(s)^-1 X, applied before the SVD;
* pillar 1 ("Mathematical Outlier Factorization"): a rank-r factorisation
  L1 L2 with r << min(d_in, d_out) carries the outliers in high precision;
  the "Step 1" decomposer splits the singular values evenly between the two
  factors (U sqrt(S), sqrt(S) V^T) and quantises what is left of the weight.

Readings (the pages leave these open; each is listed in the design notes):
* smoothing factor s_k = max_m |Xcal_mk|^alpha / max_n |W_nk|^(1-alpha)
  (the SmoothQuant form; the pages give only the transform), alpha = 0.5,
  clamped to [1e-4, 1e4]; an all-zero channel gets s_k = 1;
* the SVD is of the smoothed weight W~ = W diag(s) and the residual is
  R = W~ - A~ B~ (the pages' three descriptions of what is factorised
  disagree; this is the plainest one that keeps W~ = A~ B~ + R exact);
* in the token-major convention (Y = X W^T) the low-rank branch is X L1 L2
  with L1 = diag(1/s) B~^T [K, r] and L2 = A~^T [r, N]; both are stored
  transposed (L1t = L1^T [r, K], L2t = L2^T [N, r]) and rounded to bf16.
"""
from __future__ import annotations

import numpy as np


def smoothing_factors(x_cal: np.ndarray, w: np.ndarray, alpha: float = 0.5) -> np.ndarray:
    """s [K] in fp64 from a calibration activation [Mc, K] and the weight [N, K]."""
    ax = np.abs(np.asarray(x_cal, np.float64)).max(axis=0)
    aw = np.abs(np.asarray(w, np.float64)).max(axis=0)
    with np.errstate(divide="ignore", invalid="ignore"):
        s = ax ** alpha / aw ** (1.0 - alpha)
    s = np.where((ax > 0) & (aw > 0) & np.isfinite(s), s, 1.0)
    return np.clip(s, 1e-4, 1e4)


def truncated_svd(a: np.ndarray, r: int, exact: bool | None = None, seed: int = 0):
    """Top-r singular triplets of ``a`` (fp64): (U_r, S_r, Vt_r).

    Small matrices use the full LAPACK SVD.  Large ones use a randomised range
    finder with oversampling and power iterations (Halko, Martinsson & Tropp,
    2011), which returns a rank-r factorisation just as exact in structure
    (W~ = A~ B~ + R holds to rounding whatever the factors are).
    """
    a = np.asarray(a, np.float64)
    if exact is None:
        exact = a.shape[0] * a.shape[1] <= 4_000_000
    if exact:
        u, s, vt = np.linalg.svd(a, full_matrices=False)
        return u[:, :r], s[:r], vt[:r, :]
    rng = np.random.Generator(np.random.PCG64(seed))
    k = min(r + 16, min(a.shape))
    omega = rng.standard_normal((a.shape[1], k))
    q, _ = np.linalg.qr(a @ omega)
    for _ in range(2):
        q, _ = np.linalg.qr(a.T @ q)
        q, _ = np.linalg.qr(a @ q)
    b = q.T @ a
    ub, s, vt = np.linalg.svd(b, full_matrices=False)
    return (q @ ub)[:, :r], s[:r], vt[:r, :]


def to_bf16_values(a: np.ndarray) -> np.ndarray:
    """Round fp64/fp32 values to the nearest bf16 (ties to even), returned as fp32."""
    f = np.ascontiguousarray(np.asarray(a, np.float32))
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32).reshape(f.shape)


def svdquant_prepare(w: np.ndarray, x_cal: np.ndarray, r: int, alpha: float = 0.5,
                     exact_svd: bool | None = None, seed: int = 0):
    """Smoothing + truncated SVD + residual for one linear.

    Returns a dict with
      inv_s [K] fp32       reciprocal smoothing factors, fl32(1/s)
      L1t  [r, K] fp32     bf16 values of (diag(1/s) B~^T)^T
      L2t  [N, r] fp32     bf16 values of A~
      R    [N, K] fp32     residual W~ - A~ B~, rounded once to fp32
      s    [K] fp64
    """
    w = np.asarray(w, np.float64)
    s = smoothing_factors(x_cal, w, alpha)
    inv_s = (np.float32(1.0) / s.astype(np.float32)).astype(np.float32)
    w_s = w * s[None, :]
    if r > 0:
        u, sv, vt = truncated_svd(w_s, r, exact_svd, seed)
        a_t = u * np.sqrt(sv)[None, :]              # A~ [N, r]
        b_t = np.sqrt(sv)[:, None] * vt             # B~ [r, K]
        resid = w_s - a_t @ b_t
        L1t = to_bf16_values(b_t / s[None, :])      # (diag(1/s) B~^T)^T
        L2t = to_bf16_values(a_t)
    else:
        resid = w_s
        L1t = np.zeros((0, w.shape[1]), np.float32)
        L2t = np.zeros((w.shape[0], 0), np.float32)
    return {"inv_s": inv_s, "L1t": L1t, "L2t": L2t,
            "R": resid.astype(np.float32), "s": s}
