"""GPU parity for inner dimensions that are a multiple of one FP4 MMA K-step
(64 elements, four 16-element scale blocks) but not of the GEMM's 256-deep
pipeline stage: the last stage is partial, and TMA fills the codes and scale
atoms past K with zeros, which add nothing to the accumulator.

Codes, scale bytes and the tensor scale are compared with the oracle bit for
bit, Y on every element within the parity tolerance.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4
from synth import make_linear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


@pytest.mark.parametrize("M,K,N,r", [
    (300, 3136, 384, 32),    # 12 full 256-deep steps + one 64-deep step; ragged rows
    (300, 320, 264, 32),     # one full step + a 64-deep one; N not a multiple of the tile
    (4608, 3136, 1024, 16),  # CTA pairs, rank 16
    (128, 192, 520, 0),      # a single partial step, a single row block, no low-rank branch
    (257, 64, 136, 32),      # K = one MMA K-step
])
def test_k_not_multiple_of_256(w4, M, K, N, r):
    import torch
    c = make_linear("kstep", M, K, N, r=r, act="student_t", bias_std=0.01, seed=900 + K)
    p = prepare(c)
    pw = w4.pack_weight(to_dev_f32(p["R"]))
    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, N, K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]) if r else None,
                        to_dev_bf16(p["L2t"]) if r else None, to_dev_bf16(c.bias))
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w if r else None)
    Y = w4.gemm(qa, w)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    # the weight the GPU packed is the oracle's, byte for byte
    assert float(w.t_w.cpu()[0]) == float(p["t_w"])
    np.testing.assert_array_equal(w.Wq.cpu().numpy(), p["Wq"])
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(w.Wsf.cpu().numpy(), N, K)[:N], p["Wsf"])
    y_ref, aux = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"],
                                     p["L1t"] if r else None, p["L2t"] if r else None, c.bias)
    assert float(qa.t_x.cpu()[0]) == float(aux["t_x"])
    np.testing.assert_array_equal(qa.Xq.cpu().numpy(), aux["xq"])
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K)[:M], aux["xsf"])
    check_y(from_dev_bf16(Y), y_ref)
