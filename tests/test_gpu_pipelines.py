"""Full-size parity of the multi-linear workloads on sampled outputs.

* Single-stream DiT MLP at 1024px (M = 4608): up-projection 3072 -> 12288
  with the GELU-tanh epilogue, then the down-projection 12288 -> 3072.
* Denoising trajectory (hidden 3072, batch 1, 2 and 4): the fused QKV +
  MLP-up linear (one smoothing vector, one activation quantisation, two GEMMs
  over row slices of one packed weight) at several steps whose outlier
  channels and magnitudes are redrawn per step, so the tensor scale changes
  every step; every code and scale byte of each step's activation is checked;
  at batch 2 and 4 also the MLP-down linear.

The per-tensor activation scale couples all rows, so the oracle computes the
whole tensor's amax and then only the sampled rows, against the weight rows of
the sampled output channels; the GPU packs the full weights and the sampled
rows of its packing are checked byte for byte first.  Every oracle input is
synthetic or oracle-computed: the down-projection is fed an oracle-computed
GELU-shaped activation, not the GPU's own output.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import gelu as ogelu
from oracle import linear as olinear
from oracle import nvfp4, prep
from synth import bf16_round, config_cases, make_linear, rng, trajectory_step_activation
from synth.inputs import act_student_t

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def gpu_weight(w4, p, bias, check_rows):
    """GPU-pack the oracle's residual; check sampled rows against the oracle;
    return (PackedWeight on device, oracle bytes of the sampled rows)."""
    import torch
    N, K = p["R"].shape
    pw = w4.pack_weight(to_dev_f32(p["R"]), inv_s=to_dev_f32(p["inv_s"]), L1t=to_dev_bf16(p["L1t"]),
                        L2t=to_dev_bf16(p["L2t"]), bias=None if bias is None else to_dev_bf16(bias))
    torch.cuda.synchronize()
    codes, osf, ot, _ = nvfp4.quantize(p["R"][check_rows], amax=np.max(np.abs(p["R"])))
    oq = nvfp4.pack(codes)
    assert float(pw.t_w.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(pw.Wq.cpu().numpy()[check_rows], oq)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(pw.Wsf.cpu().numpy(), N, K)[check_rows], osf)
    return pw, oq, osf, ot


def oracle_sampled(x, p, oq, osf, ot, bias, rows, cols, gelu=False):
    y, aux = olinear.w4a4_linear(x, p["inv_s"], oq, osf, ot, p["L1t"], p["L2t"][cols],
                                 None if bias is None else bias[cols], rows=rows)
    return (ogelu.gelu_tanh(y) if gelu else y), aux


def gelu_shaped_activation(M, K, seed):
    """bf16(GELU(z)) with z drawn like a projection output (N(0,1) with 1%
    heavy-tailed channels): the distribution a down-projection sees."""
    z, _ = act_student_t(rng(seed), M, K, scale=8.0)
    return bf16_round(ogelu.gelu_tanh(z).astype(np.float32))


def test_mlp_block_1024px(w4):
    import torch
    up, down = config_cases(3)
    g = rng(33)
    rows = np.sort(g.choice(up.M, 192, replace=False))
    cols_up = np.sort(g.choice(up.N, 512, replace=False))
    cols_dn = np.sort(g.choice(down.N, 512, replace=False))

    # up-projection with the GELU epilogue
    p_up = prep.svdquant_prepare(up.w, up.x_cal, up.r, up.alpha)
    w_up, oq, osf, ot = gpu_weight(w4, p_up, up.bias, cols_up)
    H = w4.linear(to_dev_bf16(up.x), w_up, epilogue=w4.EPI_GELU_TANH)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    h = from_dev_bf16(H)
    ref, _ = oracle_sampled(up.x, p_up, oq, osf, ot, up.bias, rows, cols_up, gelu=True)
    check_y(h[rows][:, cols_up], ref)

    # down-projection on a GELU-shaped activation of the same shape
    x_dn = gelu_shaped_activation(down.M, down.K, 3003)
    x_cal = gelu_shaped_activation(512, down.K, 3503)
    p_dn = prep.svdquant_prepare(down.w, x_cal, down.r, down.alpha)
    w_dn, oq, osf, ot = gpu_weight(w4, p_dn, down.bias, cols_dn)
    qa = w4.quantize_act(to_dev_bf16(x_dn), w_dn.inv_s, w_dn.L1t, w_dn.t_w)
    Y = w4.gemm(qa, w_dn)
    torch.cuda.synchronize()
    y = from_dev_bf16(Y)
    ref, aux = oracle_sampled(x_dn, p_dn, oq, osf, ot, down.bias, rows, cols_dn)
    assert float(qa.t_x.cpu()[0]) == float(aux["t_x"])
    np.testing.assert_array_equal(qa.Xq.cpu().numpy()[rows], aux["xq"])
    check_y(y[rows][:, cols_dn], ref)


def test_denoising_trajectory_fused_qkv_mlp(w4):
    import torch
    qkv, mlp, _down = config_cases(5)
    K = qkv.K
    n_qkv = qkv.N
    # the fused projection's weight and bias; calibration spread over the schedule
    w = np.concatenate([qkv.w, mlp.w], axis=0)
    bias = np.concatenate([qkv.bias, mlp.bias])
    x_cal = np.concatenate([trajectory_step_activation(t, 10, K)[0] for t in range(50)], axis=0)
    p = prep.svdquant_prepare(w, x_cal, 32, 0.5)
    g = rng(55)
    cols = np.sort(g.choice(w.shape[0], 768, replace=False))
    pw, oq, osf, ot = gpu_weight(w4, p, bias, cols)
    w_qkv, w_mlp = pw.rows(0, n_qkv), pw.rows(n_qkv, w.shape[0])
    c_qkv = cols[cols < n_qkv]
    c_mlp = cols[cols >= n_qkv]
    t_prev = None
    for step in (0, 25, 49):
        x, meta = trajectory_step_activation(step, 4608, K)
        rows = np.sort(rng(100 + step).choice(4608, 128, replace=False))
        qa = w4.quantize_act(to_dev_bf16(x), pw.inv_s, pw.L1t, pw.t_w)
        Yq = w4.gemm(qa, w_qkv)
        Hm = w4.gemm(qa, w_mlp, epilogue=w4.EPI_GELU_TANH)
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0
        yq, hm = from_dev_bf16(Yq), from_dev_bf16(Hm)
        sel_q = np.searchsorted(cols, c_qkv)
        sel_m = np.searchsorted(cols, c_mlp)
        ref_q, aux = olinear.w4a4_linear(x, p["inv_s"], oq[sel_q], osf[sel_q], ot, p["L1t"], p["L2t"][c_qkv],
                                         bias[c_qkv], rows=rows)
        ref_m, _ = olinear.w4a4_linear(x, p["inv_s"], oq[sel_m], osf[sel_m], ot, p["L1t"], p["L2t"][c_mlp],
                                       bias[c_mlp], rows=rows)
        t_x = float(qa.t_x.cpu()[0])
        assert t_x == float(aux["t_x"])
        assert check_activation_bytes(qa, x, p["inv_s"]) == t_x
        assert t_x != t_prev, "the activation scale is recomputed every step"
        t_prev = t_x
        check_y(yq[rows][:, c_qkv], ref_q)
        check_y(hm[rows][:, c_mlp - n_qkv], ogelu.gelu_tanh(ref_m))


def check_activation_bytes(qa, x, inv_s, chunk=4096):
    """Every code and scale byte of a quantised activation against the oracle
    (row chunks under the whole tensor's amax); returns the tensor scale."""
    M, K = x.shape
    amax = np.float32(0.0)
    for r0 in range(0, M, chunk):
        amax = max(amax, np.float32(np.max(np.abs(nvfp4.smooth(x[r0:r0 + chunk], inv_s)))))
    t_x = float(qa.t_x.cpu()[0])
    assert t_x == float(nvfp4.tensor_scale(amax))
    gq = qa.Xq.cpu().numpy()
    gsf = sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K)
    for r0 in range(0, M, chunk):
        codes, sf, _, _ = nvfp4.quantize(nvfp4.smooth(x[r0:r0 + chunk], inv_s), amax=amax)
        np.testing.assert_array_equal(gq[r0:r0 + chunk], nvfp4.pack(codes), err_msg=f"codes, rows from {r0}")
        np.testing.assert_array_equal(gsf[r0:r0 + chunk], sf, err_msg=f"scales, rows from {r0}")
    return t_x


@pytest.mark.parametrize("B", [2, 4])
def test_denoising_trajectory_batches(w4, B):
    """The denoising block at batch B (M = 4608 B tokens, every image its own
    draw at the step's outlier schedule): the fused QKV + MLP-up linear at
    steps 0, 25 and 49 with every activation code and scale byte checked, Y
    sampled; and the MLP-down linear (12288 -> 3072) on a GELU-shaped
    activation of the same batch."""
    import torch
    qkv, mlp, down = config_cases(5)
    K = qkv.K
    n_qkv = qkv.N
    M = 4608 * B
    w = np.concatenate([qkv.w, mlp.w], axis=0)
    bias = np.concatenate([qkv.bias, mlp.bias])
    x_cal = np.concatenate([trajectory_step_activation(t, 10, K)[0] for t in range(50)], axis=0)
    p = prep.svdquant_prepare(w, x_cal, 32, 0.5)
    g = rng(56 + B)
    cols = np.sort(g.choice(w.shape[0], 512, replace=False))
    pw, oq, osf, ot = gpu_weight(w4, p, bias, cols)
    w_qkv, w_mlp = pw.rows(0, n_qkv), pw.rows(n_qkv, w.shape[0])
    c_qkv, c_mlp = cols[cols < n_qkv], cols[cols >= n_qkv]
    sel_q, sel_m = np.searchsorted(cols, c_qkv), np.searchsorted(cols, c_mlp)
    t_prev = None
    for step in (0, 25, 49):
        x, _ = trajectory_step_activation(step, M, K)
        rows = np.sort(rng(200 + step).choice(M, 96, replace=False))
        qa = w4.quantize_act(to_dev_bf16(x), pw.inv_s, pw.L1t, pw.t_w)
        Yq = w4.gemm(qa, w_qkv)
        Hm = w4.gemm(qa, w_mlp, epilogue=w4.EPI_GELU_TANH)
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0
        t_x = check_activation_bytes(qa, x, p["inv_s"])
        assert t_x != t_prev, "the activation scale is recomputed every step"
        t_prev = t_x
        idx = torch.from_numpy(rows).cuda()
        yq, hm = from_dev_bf16(Yq[idx]), from_dev_bf16(Hm[idx])
        ref_q, _ = olinear.w4a4_linear(x, p["inv_s"], oq[sel_q], osf[sel_q], ot, p["L1t"], p["L2t"][c_qkv],
                                       bias[c_qkv], rows=rows)
        ref_m, _ = olinear.w4a4_linear(x, p["inv_s"], oq[sel_m], osf[sel_m], ot, p["L1t"], p["L2t"][c_mlp],
                                       bias[c_mlp], rows=rows)
        check_y(yq[:, c_qkv], ref_q)
        check_y(hm[:, c_mlp - n_qkv], ogelu.gelu_tanh(ref_m))
        del Yq, Hm, qa

    # MLP-down at the same batch
    x_dn = gelu_shaped_activation(M, down.K, 5100 + B)
    p_dn = prep.svdquant_prepare(down.w, gelu_shaped_activation(512, down.K, 5600 + B), down.r, down.alpha)
    cols_dn = np.sort(rng(57 + B).choice(down.N, 384, replace=False))
    w_dn, oq_d, osf_d, ot_d = gpu_weight(w4, p_dn, down.bias, cols_dn)
    qa = w4.quantize_act(to_dev_bf16(x_dn), w_dn.inv_s, w_dn.L1t, w_dn.t_w)
    Y = w4.gemm(qa, w_dn)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    check_activation_bytes(qa, x_dn, p_dn["inv_s"])
    rows = np.sort(rng(300 + B).choice(M, 96, replace=False))
    y = from_dev_bf16(Y[torch.from_numpy(rows).cuda()])[:, cols_dn]
    ref, _ = oracle_sampled(x_dn, p_dn, oq_d, osf_d, ot_d, down.bias, rows, cols_dn)
    check_y(y, ref)
