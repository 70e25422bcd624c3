"""Offline SVDQuant preparation of a linear layer's weight (runs once per
weight, never on the per-step hot path).

Steps ("SVDQuant Guide: 4-Bit DiT Acceleration & Outlier Absorption"):
1. smoothing factors s_k = max|Xcal_k|^alpha / max|W_k|^(1-alpha), clamped to
   [1e-4, 1e4] (pillar 2, "SmoothQuant Pre-Conditioning for DiTs"; the
   SmoothQuant form of s is this library's reading, the page gives only the
   transform W' = W diag(s), X' = diag(s)^-1 X);
2. a rank-r factorisation W~ = W diag(s) ~ A~ B~ with the singular values split
   evenly between the factors (pillar 1 and the page's "Step 1" decomposer),
   computed here with a randomised truncated SVD;
3. the residual R = W~ - A~ B~ is packed to NVFP4 by the library's
   ``nvfp4_pack_weight`` kernel; L1t = B~ diag(1/s) and L2t = A~ are kept in bf16.

Dense linear algebra of this one-off step uses PyTorch's library routines on
the GPU; the packing itself runs in the library's own kernel.
"""
from __future__ import annotations

import torch

from . import PackedWeight, pack_weight


def smoothing_factors(x_cal: torch.Tensor, w: torch.Tensor, alpha: float = 0.5) -> torch.Tensor:
    ax = x_cal.abs().amax(dim=0).double()
    aw = w.abs().amax(dim=0).double()
    s = ax.pow(alpha) / aw.pow(1.0 - alpha)
    ok = (ax > 0) & (aw > 0) & torch.isfinite(s)
    s = torch.where(ok, s, torch.ones_like(s))
    return s.clamp(1e-4, 1e4)


def svdquant_prepare(w: torch.Tensor, x_cal: torch.Tensor, r: int = 32, alpha: float = 0.5,
                     bias: torch.Tensor | None = None, niter: int = 2, seed: int = 0) -> PackedWeight:
    """Prepare one linear (weight [N, K] on the GPU) for ``linear``/``gemm``."""
    s = smoothing_factors(x_cal, w, alpha)
    inv_s = (1.0 / s.float()).contiguous()
    w_s = w.double() * s[None, :]
    if r > 0:
        gen_state = torch.random.get_rng_state()
        torch.manual_seed(seed)
        u, sv, v = torch.svd_lowrank(w_s, q=min(r + 16, min(w_s.shape)), niter=niter)
        torch.random.set_rng_state(gen_state)
        root = sv[:r].sqrt()
        a = u[:, :r] * root[None, :]            # A~ [N, r]
        b = root[:, None] * v[:, :r].T          # B~ [r, K]
        resid = (w_s - a @ b).float().contiguous()
        L1t = (b / s[None, :]).to(torch.bfloat16).contiguous()
        L2t = a.to(torch.bfloat16).contiguous()
    else:
        resid = w_s.float().contiguous()
        L1t = L2t = None
    packed = pack_weight(resid, inv_s=inv_s, L1t=L1t, L2t=L2t,
                         bias=None if bias is None else bias.to(torch.bfloat16).contiguous())
    return packed


def swiglu_row_order(n_plain: int, n_ff: int, device=None) -> torch.Tensor:
    """Row order that ``w4a4_gemm_swiglu`` expects for a fused projection
    whose weight is laid out [plain (n_plain rows) | gate (n_ff) | up (n_ff)]:
    the plain rows, then per block of 16 features its 16 gate rows followed
    by its 16 up rows.  Apply it to the weight (and bias) before
    ``svdquant_prepare``: a row permutation leaves the smoothing factors and
    the singular values unchanged and permutes the residual and L2t rows."""
    if n_ff % 16:
        raise ValueError("n_ff must be a multiple of 16")
    blocks = torch.arange(n_ff // 16, device=device)[:, None]
    i = torch.arange(16, device=device)[None, :]
    gate = n_plain + 16 * blocks + i
    up = n_plain + n_ff + 16 * blocks + i
    tail = torch.cat([gate, up], dim=1).reshape(-1)
    return torch.cat([torch.arange(n_plain, device=device), tail])


def rope_table(pos: torch.Tensor, axes_dims, base: float = 10000.0) -> torch.Tensor:
    """The table ``w4a4_gemm_rope`` reads, from integer token positions ``pos``
    [M, n_axes]: per token, the (cos, sin) of each head feature pair,
    interleaved, fp32 [M, sum(axes_dims)].  Axis a owns the next
    axes_dims[a] / 2 pairs; pair j of the axis turns at base^(-2j /
    axes_dims[a]) per unit of that axis's position (one axis: the rotary
    embedding's usual schedule).  Built once per sequence layout, in fp64 and
    rounded once to fp32, like the precomputed position embedding of a DiT."""
    pos = pos.to(torch.float64)
    if pos.dim() == 1:
        pos = pos[:, None]
    if pos.shape[1] != len(axes_dims) or any(d % 2 for d in axes_dims):
        raise ValueError("one even feature count per position axis")
    theta = torch.cat([pos[:, a:a + 1] * torch.pow(torch.tensor(float(base), dtype=torch.float64, device=pos.device),
                                                   -torch.arange(0, d, 2, dtype=torch.float64, device=pos.device) / d)
                       for a, d in enumerate(axes_dims)], dim=1)
    return torch.stack([torch.cos(theta), torch.sin(theta)], dim=-1).reshape(pos.shape[0], -1).to(torch.float32)
