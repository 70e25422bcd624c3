"""The GELU-tanh epilogue, checked on its own, element by element.

With a zero activation the quantiser writes zero codes and zero scales with
t_x = 1, the low-rank term is 0, so the GEMM's output is GELU(bias[n]) rounded
to bf16 in every row.  A sweep of bias values therefore probes the
epilogue's GELU against the oracle's fp64 formula
0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))):

* within one bf16 ulp for y >= -5.5, where the fp64 formula itself keeps at
  least seven significant digits (1 + tanh(u) > 1e-8 there);
* for y < -5.5 (|GELU(y)| < 6e-9, where the fp64 formula loses its relative
  accuracy to cancellation) the output is non-positive and no larger in
  magnitude than at -5.5.

Both GEMM kernels: M = 64 (single CTA) and M = 300 (CTA pairs, ragged M).
"""
import numpy as np
import pytest

from helpers import from_dev_bf16, to_dev_bf16, to_dev_f32
from oracle import gelu as ogelu
from oracle import nvfp4
from synth import bf16_round, rng

pytestmark = pytest.mark.gpu

N, K = 3072, 256
TAIL = -5.5


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def bias_sweep():
    g = rng(31)
    special = np.array([0.0, -0.0, 1e-30, -1e-30, 1e-8, -1e-8, 1e-3, -1e-3, 0.5, -0.5, 1.0, -1.0,
                        3.0, -3.0, 100.0, 1e4, -20.0, -40.0, -1e4], np.float32)
    dense = np.linspace(TAIL, 12.0, 2048, dtype=np.float32)
    tail = np.linspace(-60.0, TAIL, 512, dtype=np.float32)
    small = (g.standard_normal(N - special.size - dense.size - tail.size) * 0.05).astype(np.float32)
    b = bf16_round(np.concatenate([special, dense, tail, small]))
    assert b.size == N
    return b


def ordered(v):
    """bf16 values as integers in ulp order (sign-magnitude -> two's complement)."""
    bits = (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.int64)
    mag = bits & 0x7FFF
    return np.where(bits & 0x8000, -mag, mag)


@pytest.mark.parametrize("M", [64, 300])
def test_gelu_epilogue_against_formula(w4, M):
    import torch
    b = bias_sweep()
    w = (rng(32).standard_normal((N, K)) * 0.02).astype(np.float32)
    wq, wsf, tw, _ = nvfp4.quantize_activation(w, None)
    sfr = np.zeros((N, K // 16), np.uint8)
    sfr[:] = wsf
    atoms = sfr.reshape(N // 128, 4, 32, K // 64, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    pw = w4.PackedWeight(torch.from_numpy(wq).cuda(), torch.from_numpy(np.ascontiguousarray(atoms)).cuda(),
                         to_dev_f32(np.array([tw], np.float32)), N, K, None, None, None, to_dev_bf16(b))
    X = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    qa = w4.quantize_act(X)
    Y = w4.gemm(qa, pw, epilogue=w4.EPI_GELU_TANH)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    assert float(qa.t_x.cpu()[0]) == 1.0
    y = from_dev_bf16(Y)
    assert np.all(y == y[0:1]), "every row holds GELU(bias)"
    got = y[0]
    ref = ogelu.gelu_tanh(b.astype(np.float64))
    near = b >= TAIL
    diff = np.abs(ordered(got[near]) - ordered(bf16_round(ref[near].astype(np.float32))))
    assert diff.max() <= 1, f"max {diff.max()} bf16 ulps at bias {b[near][np.argmax(diff)]}"
    # zero bias: y = alpha * (+0) + (+/-0) = +0 in round-to-nearest, GELU(+0) = +0
    assert got[0] == 0.0 and got[1] == 0.0
    far = ~near
    bound = abs(ogelu.gelu_tanh(np.array([TAIL]))[0])
    assert np.all(got[far] <= 0.0) and np.all(np.abs(got[far]) <= bound)
