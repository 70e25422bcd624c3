"""GPU parity of the quantising epilogue (w4a4_gemm_quantize_next): the
GEMM writes the next layer's NVFP4 codes and scale bytes of its outputs
under a given tensor scale.

* Exact operands: grid-valued codes with a 6 in every block quantise to
  themselves, so the accumulator is exact; the epilogue's value is then
  bf16(fl32(fl32(t_x t_w) acc)) (no bias), which the test forms from the
  oracle's exact product in that precision.  The next layer's codes and
  scale bytes must equal the oracle's quantisation of it, given the tensor
  scale, byte for byte (no value from the GPU enters the expected bytes).
* Realistic inputs (GELU epilogue; SwiGLU outputs written into a wider next
  activation at a column offset): the bf16 outputs match the oracle within
  the parity tolerance, and the codes and scale bytes are exactly the NVFP4
  quantisation, under the given scale, of the outputs the kernel stored (a
  property of the result), columns outside the written range untouched; with
  the bf16 store switched off the codes are the same.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import gelu as ogelu
from oracle import linear as olinear
from oracle import nvfp4, prep
from oracle import swiglu as oswiglu
from synth import make_linear, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def upload_weight(w4, p, N, K, bias=None, perm=None):
    import torch
    R = p["R"] if perm is None else p["R"][perm]
    pw = w4.pack_weight(to_dev_f32(R))
    torch.cuda.synchronize()
    r = 0 if p["L1t"] is None or len(p["L1t"]) == 0 else p["L1t"].shape[0]
    L2t = None if r == 0 else (p["L2t"] if perm is None else p["L2t"][perm])
    return w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, N, K, to_dev_f32(p["inv_s"]),
                           None if r == 0 else to_dev_bf16(p["L1t"]), None if r == 0 else to_dev_bf16(L2t),
                           None if bias is None else to_dev_bf16(bias if perm is None else bias[perm]))


def expected_codes(y_bf16, inv_s, t):
    """The oracle's NVFP4 quantisation of a bf16 activation under tensor scale t."""
    codes, sf, _, _ = nvfp4.quantize(nvfp4.smooth(y_bf16, inv_s), t=t)
    return nvfp4.pack(codes), sf


def test_exact_operands(w4):
    import torch
    g = rng(81)
    M, K, N = 300, 512, 384
    grid = np.array(nvfp4.E2M1_VALUES[:8], np.float32)
    x = (grid[g.integers(0, 8, (M, K))] * g.choice([-1, 1], (M, K))).astype(np.float32)
    wv = (grid[g.integers(0, 8, (N, K))] * g.choice([-1, 1], (N, K))).astype(np.float32)
    x[:, ::16] = 6.0
    wv[:, ::16] = -6.0
    p = {"R": wv, "inv_s": np.ones(K, np.float32), "L1t": None, "L2t": None}
    w = upload_weight(w4, p, N, K)
    qa = w4.quantize_act(to_dev_bf16(x), None)
    s_next = (1.0 / np.exp(0.3 * g.standard_normal(N))).astype(np.float32)
    t_next = np.float32(0.0123)
    Y, _, nq, nsf = w4.gemm_quantize_next(qa, w, to_dev_f32(np.array([t_next], np.float32)),
                                          next_inv_s=to_dev_f32(s_next))
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    # the epilogue's value in its own precision, from the oracle's exact product
    _, sx, tx, _ = nvfp4.quantize_activation(x, None)
    _, sw, tw, _ = nvfp4.quantize_activation(wv, None)
    assert float(qa.t_x.cpu()[0]) == float(tx) and float(w.t_w.cpu()[0]) == float(tw)
    # every block scale is 448 and every code its value, so the accumulator
    # (the sum of decoded code x scale products) is 448^2 x the exact product
    assert (sx == 0x7E).all() and (sw == 0x7E).all()
    acc = (x.astype(np.float64) @ wv.astype(np.float64).T) * (448.0 * 448.0)
    acc32 = acc.astype(np.float32)
    assert np.array_equal(acc32.astype(np.float64), acc)
    y32 = (np.float32(np.float32(tx) * np.float32(tw)) * acc32).astype(np.float32) + np.float32(0.0)
    y_bf16 = prep.to_bf16_values(y32)
    np.testing.assert_array_equal(from_dev_bf16(Y), y_bf16)
    oq, osf = expected_codes(y_bf16, s_next, t_next)
    np.testing.assert_array_equal(nq.cpu().numpy(), oq)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(nsf.cpu().numpy(), M, N)[:M], osf)


@pytest.mark.parametrize("M,K,N", [(300, 512, 1024), (4608, 3072, 12288)])
def test_gelu_outputs_quantised(w4, M, K, N):
    import torch
    c = make_linear("up", M, K, N, r=32, act="student_t", bias_std=0.01, seed=M + N + 5)
    p = prepare(c)
    w = upload_weight(w4, p, N, K, c.bias)
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    s_next = (1.0 / np.exp(0.3 * rng(9).standard_normal(N))).astype(np.float32)
    t_next = np.float32(0.0021)
    t_dev = to_dev_f32(np.array([t_next], np.float32))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y, _, nq, nsf = w4.gemm_quantize_next(qa, w, t_dev, next_inv_s=to_dev_f32(s_next), epilogue=w4.EPI_GELU_TANH,
                                          next_amax=amax)
    _, _, nq2, nsf2 = w4.gemm_quantize_next(qa, w, t_dev, next_inv_s=to_dev_f32(s_next),
                                            epilogue=w4.EPI_GELU_TANH, store_outputs=False)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y = from_dev_bf16(Y)
    rows = np.sort(rng(10).choice(M, min(M, 128), replace=False))
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"], c.bias,
                                   rows=rows)
    check_y(y[rows], ogelu.gelu_tanh(y_ref))
    oq, osf = expected_codes(y, s_next, t_next)                     # property of the stored output
    np.testing.assert_array_equal(nq.cpu().numpy(), oq)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(nsf.cpu().numpy(), M, N)[:M], osf)
    assert torch.equal(nq, nq2) and torch.equal(nsf, nsf2)         # the bf16 store changes nothing
    assert float(amax.cpu()[0]) == float(np.max(np.abs((y * s_next[None, :]).astype(np.float32))))


def test_swiglu_outputs_into_a_wider_activation(w4):
    """SwiGLU outputs H quantised into columns [64, 64 + 384) of a 512-wide
    next activation, as the 2048px block's output projection sees
    [attention | H]."""
    import torch
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    M, K, n_plain, n_ff = 300, 512, 256, 384
    N = n_plain + 2 * n_ff
    next_K, next_col = 512, 64
    c = make_linear("fused", M, K, N, r=32, act="student_t", bias_std=0.5, seed=91)
    p = prepare(c)
    perm = gprep.swiglu_row_order(n_plain, n_ff).numpy()
    w = upload_weight(w4, p, N, K, c.bias, perm)
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    s_next = (1.0 / np.exp(0.3 * rng(11).standard_normal(n_ff))).astype(np.float32)
    t_next = np.float32(0.017)
    nq = torch.full((M, next_K // 2), 0xAB, dtype=torch.uint8, device="cuda")
    nsf = torch.full((w4.nvfp4_sf_bytes(M, next_K),), 0xCD, dtype=torch.uint8, device="cuda")
    Y, H, _, _ = w4.gemm_quantize_next(qa, w, to_dev_f32(np.array([t_next], np.float32)),
                                       next_inv_s=to_dev_f32(s_next), n_plain=n_plain, next_K=next_K,
                                       next_col=next_col, next_q=nq, next_sf=nsf)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"], c.bias)
    plain_ref, h_ref = oswiglu.split_fused(y_ref, n_plain, n_ff)
    h = from_dev_bf16(H)
    check_y(h, h_ref)
    check_y(from_dev_bf16(Y), plain_ref)
    oq, osf = expected_codes(h, s_next, t_next)
    got_q = nq.cpu().numpy()
    got_sf = sf_atoms_to_rowmajor(nsf.cpu().numpy(), M, next_K)
    np.testing.assert_array_equal(got_q[:, next_col // 2:(next_col + n_ff) // 2], oq)
    np.testing.assert_array_equal(got_sf[:M, next_col // 16:(next_col + n_ff) // 16], osf)
    # the rest of the next activation is untouched
    assert (got_q[:, :next_col // 2] == 0xAB).all() and (got_q[:, (next_col + n_ff) // 2:] == 0xAB).all()
    assert (got_sf[:M, :next_col // 16] == 0xCD).all() and (got_sf[:M, (next_col + n_ff) // 16:] == 0xCD).all()
