"""GPU parity of the SwiGLU epilogue (w4a4_gemm_swiglu).

A fused projection's weight is laid out [plain | gate | up]; the oracle
evaluates the layer in that natural order in fp64 and applies
silu(gate) * up to the matching columns (oracle.swiglu).  The GPU packs the
same residual rows in the kernel's order (prep.swiglu_row_order: per 16
features, the gate rows then the up rows), and its plain outputs Y and SwiGLU
outputs H must match the oracle within the parity tolerance.  The epilogue's
next-layer amax over H is checked as a property of the H it stored and
against the oracle's H.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import swiglu as oswiglu
from synth import bf16_round, make_linear, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def amax_of(x, inv_s):
    xs = (np.asarray(x, np.float32) * np.asarray(inv_s, np.float32)[None, :]).astype(np.float32)
    return np.float32(np.max(np.abs(xs)))


@pytest.mark.parametrize("M,K,n_plain,n_ff,r", [
    (300, 512, 256, 384, 32),     # ragged rows; the last tile half full
    (4608, 3072, 0, 1536, 32),    # SwiGLU only, CTA pairs over 36 row blocks
    (128, 768, 512, 256, 16),     # a single row block, rank 16
])
def test_swiglu_epilogue(w4, M, K, n_plain, n_ff, r):
    import torch
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    N = n_plain + 2 * n_ff
    c = make_linear("fused", M, K, N, r=r, act="student_t", bias_std=0.5, seed=M + N + r)
    p = prepare(c)                                    # natural row order [plain | gate | up]
    perm = gprep.swiglu_row_order(n_plain, n_ff).numpy()
    pw = w4.pack_weight(to_dev_f32(p["R"][perm]))     # the kernel's row order
    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, N, K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                        to_dev_bf16(p["L2t"][perm]), to_dev_bf16(c.bias[perm]))
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    s_next = (1.0 / np.exp(0.3 * rng(8).standard_normal(n_ff))).astype(np.float32)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y, H = w4.gemm_swiglu(qa, w, n_plain, next_inv_s=to_dev_f32(s_next), next_amax=amax)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    # the packing is the oracle's, permuted
    assert float(w.t_w.cpu()[0]) == float(p["t_w"])
    np.testing.assert_array_equal(w.Wq.cpu().numpy(), p["Wq"][perm])
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(w.Wsf.cpu().numpy(), N, K)[:N], p["Wsf"][perm])
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"], c.bias)
    plain_ref, h_ref = oswiglu.split_fused(y_ref, n_plain, n_ff)
    h = from_dev_bf16(H)
    check_y(h, h_ref)
    if n_plain:
        check_y(from_dev_bf16(Y), plain_ref)
    else:
        assert Y is None
    got = float(amax.cpu()[0])
    assert got == float(amax_of(h, s_next))          # exactly the stored H's amax
    want = float(amax_of(bf16_round(h_ref.astype(np.float32)), s_next))
    assert abs(got - want) <= 2e-2 * want

