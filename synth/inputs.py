"""Seeded synthetic activations, weights and biases shaped like FLUX DiT linears.

Shapes follow the pages' workloads: at 1024x1024 a FLUX transformer sees
4096 image tokens (a 64x64 latent after 2x2 patching) plus 512 text tokens,
hidden size 3072; the 2048x2048 case has 16384 + 512 tokens.  Activations carry
the channel outliers that the SVDQuant page describes ("a handful of channels
exhibit magnitudes exceeding 100x the median", "SVDQuant Guide: 4-Bit DiT
Acceleration & Outlier Absorption", section "Why Standard Low-Bit
Quantization Fails on DiTs"), and their outlier channels move from one
denoising step to the next (same section, "Timestep-Dynamic Activation
Drift").

Every generator takes an explicit seed and uses numpy's PCG64.  Values are
returned as float32 arrays that hold exactly representable bf16 values, plus the
raw bf16 bit patterns (uint16) for upload.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

__all__ = [
    "bf16_bits", "bf16_round", "bits_to_f32", "LinearCase", "make_linear",
    "CONFIGS", "config_cases", "trajectory_step_activation", "rng", "token_positions",
]


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs).

    Uses torch's (multi-threaded, round-to-nearest-even) cast when torch is
    importable, else the same rounding on the bit pattern in numpy."""
    f = np.ascontiguousarray(np.asarray(a, np.float32))
    try:
        import torch
        return torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    except ImportError:
        u = f.view(np.uint32)
        lsb = (u >> 16) & np.uint32(1)
        return ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(a: np.ndarray) -> np.ndarray:
    return bits_to_f32(bf16_bits(a))


# --------------------------------------------------------------------------
# activation recipes
# --------------------------------------------------------------------------

def act_normal_outliers(g, M, K, n_out, scale):
    """N(0,1) with ``n_out`` whole channels multiplied by ``scale``."""
    x = g.standard_normal((M, K), dtype=np.float32)
    ch = g.choice(K, size=n_out, replace=False) if n_out else np.zeros(0, np.int64)
    x[:, ch] *= np.float32(scale)
    return x, np.sort(ch)


def act_student_t(g, M, K, frac=0.01, nu=2.0, scale=50.0, channels=None):
    """N(0,1) with round(frac*K) channels replaced by scale * Student-t(nu)."""
    x = g.standard_normal((M, K), dtype=np.float32)
    n_out = int(round(frac * K))
    ch = channels if channels is not None else np.sort(g.choice(K, size=n_out, replace=False))
    x[:, ch] = (scale * g.standard_t(nu, size=(M, len(ch)))).astype(np.float32)
    return x, ch


def act_lognormal_channels(g, M, K, sigma=1.5, mags=None):
    """x_mk = z_mk * exp(sigma * g_k): per-channel lognormal(0, sigma) magnitudes."""
    if mags is None:
        mags = np.exp(sigma * g.standard_normal(K)).astype(np.float32)
    z = g.standard_normal((M, K), dtype=np.float32)
    return (z * mags[None, :]).astype(np.float32), mags


def trajectory_step_activation(step: int, M: int, K: int, n_out: int = 31,
                               lo: float = 20.0, hi: float = 200.0, seed_base: int = 5000):
    """Activation of one denoising step: the outlier set and its magnitude are
    re-drawn every step from seed ``seed_base + step`` (magnitude log-uniform
    in [lo, hi])."""
    g = rng(seed_base + step)
    mag = float(np.exp(g.uniform(np.log(lo), np.log(hi))))
    x, ch = act_normal_outliers(g, M, K, n_out, mag)
    return bf16_round(x), {"channels": ch, "magnitude": mag}


# --------------------------------------------------------------------------
# one linear layer's inputs
# --------------------------------------------------------------------------

@dataclass
class LinearCase:
    name: str
    M: int
    K: int
    N: int
    r: int
    x: np.ndarray            # [M, K] fp32 holding bf16 values
    w: np.ndarray            # [N, K] fp32 holding bf16 values (the bf16 master weight)
    bias: np.ndarray | None  # [N] fp32 holding bf16 values, or None
    x_cal: np.ndarray        # [Mc, K] calibration activation (separate draw)
    alpha: float = 0.5
    meta: dict = field(default_factory=dict)


def make_linear(name, M, K, N, r=32, act="normal_outliers", n_out=8, out_scale=100.0,
                bias_std=0.0, w_std=0.02, seed=0, m_cal=None, alpha=0.5):
    """Inputs for one linear: activation, bf16 weight, bias, calibration draw.

    ``act`` selects the activation recipe: "normal_outliers" (``n_out``
    channels times ``out_scale``), "student_t" (1% heavy-tailed channels,
    Student-t nu=2 times 50) or "lognormal" (per-channel lognormal(0,1.5)
    magnitudes).  The calibration draw shares the outlier channels / channel
    magnitudes with the activation but not its values.
    """
    g = rng(seed)
    gc = rng(seed + 500)
    m_cal = m_cal or min(M, 512)
    if act == "normal_outliers":
        x, ch = act_normal_outliers(g, M, K, n_out, out_scale)
        xc = gc.standard_normal((m_cal, K), dtype=np.float32)
        xc[:, ch] *= np.float32(out_scale)
        meta = {"channels": ch}
    elif act == "student_t":
        x, ch = act_student_t(g, M, K)
        xc, _ = act_student_t(gc, m_cal, K, channels=ch)
        meta = {"channels": ch}
    elif act == "lognormal":
        x, mags = act_lognormal_channels(g, M, K)
        xc, _ = act_lognormal_channels(gc, m_cal, K, mags=mags)
        meta = {"channel_mags": mags}
    else:
        raise ValueError(act)
    gw = rng(seed + 1)
    w = (w_std * gw.standard_normal((N, K), dtype=np.float32)).astype(np.float32)
    bias = None
    if bias_std > 0:
        bias = bf16_round((bias_std * gw.standard_normal(N, dtype=np.float32)).astype(np.float32))
    return LinearCase(name, M, K, N, r, bf16_round(x), bf16_round(w), bias,
                      bf16_round(xc), alpha, meta)


def token_positions(n_text: int, h: int, w: int, batch: int = 1) -> np.ndarray:
    """Integer positions [batch * (n_text + h * w), 3] of a joint text + image
    token sequence, per image: the text tokens first, all at (0, 0, 0), then
    the h x w latent patches in row-major order at (0, row, column).  Pure
    indices: no draw and no arithmetic of the method."""
    img = np.stack(np.meshgrid(np.arange(h), np.arange(w), indexing="ij"), axis=-1).reshape(-1, 2)
    one = np.concatenate([np.zeros((n_text, 3), np.int64),
                          np.concatenate([np.zeros((h * w, 1), np.int64), img], axis=1)])
    return np.tile(one, (batch, 1))


# --------------------------------------------------------------------------
# the five workload configurations
# --------------------------------------------------------------------------

CONFIGS = {
    1: "single W4A4 linear, M=128 K=3072 N=3072, 8 outlier channels x100, rank 32, bias 0",
    2: "FLUX-1024px QKV projection, M=4608 K=3072 N=9216, 1% Student-t(2)x50 channels, rank 32, bias N(0,0.01)",
    3: "single-stream DiT MLP at 1024px, M=4608: up 3072->12288, GELU-tanh, down 12288->3072",
    4: "2048px large-hidden block, M=16896: fused QKV+SwiGLU-up 6144->55296 and output 24576->6144, lognormal(0,1.5) channels",
    5: "denoising trajectory: block with hidden 3072 (QKV 9216, MLP 12288) at batch 1,2,4 over 50 steps, outliers re-drawn per step",
}


def config_cases(cfg: int, scale_m: float = 1.0, seed_base: int = 1000):
    """LinearCase list for one configuration (``scale_m`` shrinks M for tests).

    For configuration 3 the down-projection's activation is produced by the
    pipeline (GELU of the up-projection), so only its weight/bias are drawn
    here; its ``x`` is a placeholder draw of the right shape.
    """
    s = seed_base + cfg

    def m(v):
        return max(1, int(round(v * scale_m)))

    if cfg == 1:
        return [make_linear("linear", m(128), 3072, 3072, act="normal_outliers", n_out=8,
                            out_scale=100.0, bias_std=0.0, seed=s)]
    if cfg == 2:
        return [make_linear("qkv", m(4608), 3072, 9216, act="student_t", bias_std=0.01, seed=s)]
    if cfg == 3:
        return [make_linear("mlp_up", m(4608), 3072, 12288, act="student_t", bias_std=0.01, seed=s),
                make_linear("mlp_down", m(4608), 12288, 3072, act="student_t", bias_std=0.01, seed=s + 100)]
    if cfg == 4:
        return [make_linear("qkv_swiglu_up", m(16896), 6144, 55296, act="lognormal", bias_std=0.0, seed=s),
                make_linear("out", m(16896), 24576, 6144, act="lognormal", bias_std=0.0, seed=s + 100)]
    if cfg == 5:
        return [make_linear("qkv", m(4608), 3072, 9216, act="normal_outliers", n_out=31,
                            out_scale=60.0, bias_std=0.01, seed=s),
                make_linear("mlp_up", m(4608), 3072, 12288, act="normal_outliers", n_out=31,
                            out_scale=60.0, bias_std=0.01, seed=s + 100),
                make_linear("mlp_down", m(4608), 12288, 3072, act="student_t", bias_std=0.01, seed=s + 200)]
    raise ValueError(cfg)
