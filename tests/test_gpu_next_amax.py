"""The fused producer epilogue (w4a4_gemm_next_amax) and the quantiser that
takes the tensor amax as an input (nvfp4_quantize_act_with_amax).

* Given the oracle's amax, the quantiser's codes, scale bytes and tensor
  scale equal the oracle's bit for bit, on a shape the single-pass path would
  take and on one the two-pass path would take (the given amax replaces both).
* The GEMM epilogue's amax of its stored bf16 outputs (after bias and GELU),
  weighted by the next layer's 1/s: exactly max |fl(Y * s)| over the output it
  wrote (a property of the result), and within bf16 rounding of the oracle's
  fp64 outputs -- on the pair kernel (M > 128) and the single-CTA kernel.
"""
import numpy as np
import pytest

from helpers import prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import gelu as ogelu
from oracle import linear as olinear
from oracle import nvfp4
from synth import bf16_round, make_linear, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def oracle_amax(x, inv_s):
    """max |fl(x * inv_s)| in fp32, one correctly rounded product per element."""
    xs = (x.astype(np.float32) * inv_s.astype(np.float32)[None, :]).astype(np.float32)
    return np.float32(np.max(np.abs(xs)))


@pytest.mark.parametrize("M,K,r", [(300, 512, 32), (4608, 12288, 32), (257, 768, 0)])
def test_quantize_with_given_amax(w4, M, K, r):
    import torch
    g = rng(M + K)
    z = g.standard_normal((M, K)).astype(np.float32)
    z[:, g.choice(K, 8, replace=False)] *= 40.0
    x = bf16_round(ogelu.gelu_tanh(z).astype(np.float32))           # a GELU-shaped activation
    inv_s = (1.0 / np.exp(0.3 * g.standard_normal(K))).astype(np.float32)
    L1t = bf16_round((g.standard_normal((32, K)) * 0.02).astype(np.float32)) if r else None
    a = oracle_amax(x, inv_s)
    qa = w4.quantize_act(to_dev_bf16(x), to_dev_f32(inv_s), None if r == 0 else to_dev_bf16(L1t),
                         to_dev_f32(np.array([0.01], np.float32)) if r else None,
                         amax=to_dev_f32(np.array([a], np.float32)))
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    oq, osf, ot, _ = nvfp4.quantize_activation(x, inv_s)
    assert float(qa.t_x.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K)[:M], osf)
    np.testing.assert_array_equal(qa.Xq.cpu().numpy(), oq)
    if r:
        U = qa.U.float().cpu().numpy().astype(np.float64)
        alpha = np.float64(np.float32(np.float32(ot) * np.float32(0.01)))
        ref = olinear.lowrank_down(x, L1t) / alpha
        assert olinear.rel_frobenius(U[:, :32] + U[:, 32:], ref) < 1e-5


@pytest.mark.parametrize("M,K,N,gelu", [(640, 3072, 12288, True), (100, 3072, 3072, False), (300, 512, 264, True),
                                         (64, 256, 19200, True)])
def test_gemm_next_amax(w4, M, K, N, gelu):
    import torch
    c = make_linear("up", M, K, N, r=32, act="student_t", bias_std=0.01, seed=M + N)
    p = prepare(c)
    qa = w4.quantize_act(to_dev_bf16(c.x), to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                         to_dev_f32(np.array([p["t_w"]], np.float32)))
    # upload the oracle-packed weight
    rb = -(-N // 128)
    sfr = np.zeros((rb * 128, K // 16), np.uint8)
    sfr[:N] = p["Wsf"]
    atoms = sfr.reshape(rb, 4, 32, K // 64, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    w = w4.PackedWeight(torch.from_numpy(p["Wq"]).cuda(), torch.from_numpy(np.ascontiguousarray(atoms)).cuda(),
                        to_dev_f32(np.array([p["t_w"]], np.float32)), N, K, to_dev_f32(p["inv_s"]),
                        to_dev_bf16(p["L1t"]), to_dev_bf16(p["L2t"]), to_dev_bf16(c.bias))
    s_next = (1.0 / np.exp(0.3 * rng(7).standard_normal(N))).astype(np.float32)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y = w4.gemm(qa, w, epilogue=w4.EPI_GELU_TANH if gelu else w4.EPI_NONE,
                next_inv_s=to_dev_f32(s_next), next_amax=amax)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    got = float(amax.cpu()[0])
    # property of the stored output: exactly its amax under the next 1/s
    y = Y.float().cpu().numpy()
    assert got == float(oracle_amax(y, s_next))
    # against the oracle's fp64 outputs, rounded to bf16 like the stored ones
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"], c.bias)
    if gelu:
        y_ref = ogelu.gelu_tanh(y_ref)
    want = float(oracle_amax(bf16_round(y_ref.astype(np.float32)), s_next))
    assert abs(got - want) <= 2e-2 * want
