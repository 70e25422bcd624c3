"""Shared test plumbing: layout conversion of GPU outputs, device upload, and
oracle-side preparation of a linear layer's inputs.

Nothing here computes the method on the GPU side: expected values come from
``oracle``; device buffers are filled from the seeded inputs of ``synth``.
"""
from __future__ import annotations

import numpy as np

from oracle import linear as olinear
from oracle import nvfp4, prep
from synth import bf16_bits

RTOL_FROB = 2e-3        # relative Frobenius error bound on Y
ROW_MAXABS = 1e-2       # per-row max |dY| <= 1e-2 * max |Y_ref row|


def sf_atoms_to_rowmajor(atoms: np.ndarray, rows: int, K: int) -> np.ndarray:
    """SF-atom bytes (layout of include/w4a4.h) -> row-major [rows_pad, K/16]."""
    rb = -(-rows // 128)
    kg = K // 64
    a = np.asarray(atoms, np.uint8).reshape(rb, kg, 32, 4, 4)     # [rb, kg, m%32, (m/32)%4, j]
    return a.transpose(0, 3, 2, 1, 4).reshape(rb * 128, kg * 4)


def to_dev_bf16(a_f32: np.ndarray):
    import torch
    bits = bf16_bits(a_f32).view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(bits)).cuda().view(torch.bfloat16)


def to_dev_f32(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, np.float32))).cuda()


def from_dev_bf16(t) -> np.ndarray:
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32)


def prepare(case, exact_svd=None):
    """Oracle preparation of one LinearCase: smoothing, SVD, residual, packed
    residual weight.  Returns a dict of numpy arrays."""
    p = prep.svdquant_prepare(case.w, case.x_cal, case.r, case.alpha, exact_svd=exact_svd)
    wq, wsf, tw, _ = nvfp4.quantize_activation(p["R"], None)
    p.update(Wq=wq, Wsf=wsf, t_w=tw)
    return p


def check_y(y_gpu: np.ndarray, y_ref: np.ndarray):
    rel = olinear.rel_frobenius(y_gpu, y_ref)
    row = olinear.row_maxabs_ratio(y_gpu, y_ref)
    assert np.all(np.isfinite(y_gpu)), "non-finite output"
    assert rel <= RTOL_FROB, f"relative Frobenius error {rel:.3e} > {RTOL_FROB}"
    assert row <= ROW_MAXABS, f"row max-abs ratio {row:.3e} > {ROW_MAXABS}"
    return rel, row
