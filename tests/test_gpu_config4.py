"""GPU parity on the 2048px large-hidden block (the largest configuration):
the fused QKV + SwiGLU-up linear 6144 -> 55296 and the output linear
24576 -> 6144, at the full 16896 tokens and at 2112 tokens (a ragged 17th row
block), with full K and N.

* Weights: the GPU packs the whole residual; sampled rows of its packing are
  compared with the oracle's bytes under the whole residual's tensor scale.
* Activations at full size: every code byte and every scale byte of the
  16896-token activation is compared with the oracle, which quantises the
  rows in chunks under the whole tensor's amax (rows are independent once the
  tensor scale is fixed).  Both activations are too large to be co-resident,
  so they take the two-pass quantiser.
* Y: sampled tokens x sampled output channels against the oracle's fp64
  result from those same oracle bytes.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4, prep
from synth import config_cases, rng

pytestmark = pytest.mark.gpu

CHUNK = 2048  # oracle rows per chunk


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


@pytest.fixture(scope="module")
def layers(w4):
    """Both linears: the full-size case, its oracle preparation and the GPU packing."""
    import torch
    out = []
    for c in config_cases(4):
        p = prep.svdquant_prepare(c.w, c.x_cal, c.r, c.alpha)
        pw = w4.pack_weight(to_dev_f32(p["R"]))
        torch.cuda.synchronize()
        w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, c.N, c.K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                            to_dev_bf16(p["L2t"]), to_dev_bf16(c.bias) if c.bias is not None else None)
        out.append((c, p, w))
    return out


def check_weight_rows(w, p, cols):
    """Sampled rows of the GPU packing against the oracle; returns the oracle bytes."""
    oq, osf, ot, _ = nvfp4.quantize(p["R"][cols], amax=np.max(np.abs(p["R"])))
    owq = nvfp4.pack(oq)
    assert float(w.t_w.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(w.Wq.cpu().numpy()[cols], owq)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(w.Wsf.cpu().numpy(), w.N, w.K)[cols], osf)
    return owq, osf, ot


def sample(M, N, which, n_rows=96, n_cols=384):
    g = rng(4000 + which + M)
    rows = np.sort(g.choice(M, n_rows, replace=False))
    rows[-1] = M - 1
    cols = np.sort(g.choice(N, n_cols, replace=False))
    cols[-1] = N - 1
    return rows, cols


@pytest.mark.parametrize("which", [0, 1])
def test_config4_full_size(w4, layers, which):
    import torch
    c, p, w = layers[which]
    M, K = c.M, c.K
    assert M == 16896
    rows, cols = sample(M, c.N, which)
    owq, osf, ot = check_weight_rows(w, p, cols)

    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    Y = w4.gemm(qa, w)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0

    # every activation code and scale byte, in row chunks under the whole tensor's amax
    amax = np.float32(0.0)
    for r0 in range(0, M, CHUNK):
        amax = max(amax, np.float32(np.max(np.abs(nvfp4.smooth(c.x[r0:r0 + CHUNK], p["inv_s"])))))
    t_x = float(qa.t_x.cpu()[0])
    assert t_x == float(nvfp4.tensor_scale(amax))
    gq = qa.Xq.cpu().numpy()
    gsf = sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K)
    for r0 in range(0, M, CHUNK):
        codes, sf, t, _ = nvfp4.quantize(nvfp4.smooth(c.x[r0:r0 + CHUNK], p["inv_s"]), amax=amax)
        assert float(t) == t_x
        np.testing.assert_array_equal(gq[r0:r0 + CHUNK], nvfp4.pack(codes), err_msg=f"codes, rows from {r0}")
        np.testing.assert_array_equal(gsf[r0:r0 + CHUNK], sf, err_msg=f"scales, rows from {r0}")
    del gq, gsf

    y = from_dev_bf16(Y[torch.from_numpy(rows).cuda()])[:, cols]
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], owq, osf, ot, p["L1t"], p["L2t"][cols],
                                   None if c.bias is None else c.bias[cols], rows=rows)
    check_y(y, y_ref)


@pytest.mark.parametrize("which", [0, 1])
def test_config4_ragged_rows(w4, layers, which):
    """2112 tokens (16.5 row blocks) through w4a4_linear, sampled Y."""
    import torch
    c, p, w = layers[which]
    M = 2112
    x = c.x[:M]
    rows, cols = sample(M, c.N, which)
    owq, osf, ot = check_weight_rows(w, p, cols)
    Y = w4.linear(to_dev_bf16(x), w)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y = from_dev_bf16(Y)[rows][:, cols]
    y_ref, aux = olinear.w4a4_linear(x, p["inv_s"], owq, osf, ot, p["L1t"], p["L2t"][cols],
                                     None if c.bias is None else c.bias[cols], rows=rows)
    check_y(y, y_ref)


def test_config4_swiglu_full_size(w4, layers):
    """The fused projection as the block runs it: QKV (3 x 6144 plain
    features) and SwiGLU (18432 gate/up pairs) in one GEMM at 16896 tokens,
    the kernel's row order from prep.swiglu_row_order; sampled Y and H
    against the oracle in the natural order, and the epilogue's amax over H
    (the output linear's input) as a property of the whole stored H."""
    import torch
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    from oracle import swiglu as oswiglu
    c, p, _ = layers[0]
    n_plain = n_ff = 18432
    assert c.N == n_plain + 2 * n_ff
    perm = gprep.swiglu_row_order(n_plain, n_ff).numpy()
    pw = w4.pack_weight(to_dev_f32(p["R"][perm]))
    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, c.N, c.K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                        to_dev_bf16(p["L2t"][perm]), None)
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    s_next = (1.0 / np.exp(0.3 * rng(44).standard_normal(n_ff))).astype(np.float32)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y, H = w4.gemm_swiglu(qa, w, n_plain, next_inv_s=to_dev_f32(s_next), next_amax=amax)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0

    g = rng(45)
    rows = np.sort(g.choice(c.M, 64, replace=False))
    rows[-1] = c.M - 1
    pc = np.sort(g.choice(n_plain, 128, replace=False))
    hc = np.sort(g.choice(n_ff, 128, replace=False))
    hc[-1] = n_ff - 1
    cols = np.concatenate([pc, n_plain + hc, n_plain + n_ff + hc])      # natural order
    # the GPU's packing of these rows (kernel order) is the oracle's
    oq, osf, ot, _ = nvfp4.quantize(p["R"][cols], amax=np.max(np.abs(p["R"])))
    inv = np.argsort(perm)                                                # natural row -> kernel row
    assert float(pw.t_w.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(pw.Wq.cpu().numpy()[inv[cols]], nvfp4.pack(oq))
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(pw.Wsf.cpu().numpy(), c.N, c.K)[inv[cols]], osf)
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], nvfp4.pack(oq), osf, ot, p["L1t"], p["L2t"][cols], None,
                                   rows=rows)
    plain_ref = y_ref[:, :len(pc)]
    h_ref = oswiglu.swiglu(y_ref[:, len(pc):len(pc) + len(hc)], y_ref[:, len(pc) + len(hc):])
    idx = torch.from_numpy(rows).cuda()
    check_y(from_dev_bf16(Y[idx])[:, pc], plain_ref)
    check_y(from_dev_bf16(H[idx])[:, hc], h_ref)

    got = float(amax.cpu()[0])
    want = np.float32(0.0)
    for r0 in range(0, c.M, 2048):
        h = from_dev_bf16(H[r0:r0 + 2048])
        want = max(want, np.float32(np.max(np.abs((h * s_next[None, :]).astype(np.float32)))))
    assert got == float(want)


def test_config4_rope_swiglu_full_size(w4, layers):
    """The fused projection with all three epilogues at 16896 tokens: the
    rotary embedding on the 2 x 6144 query and key features (heads of 128,
    angles of the text + 128 x 128 image-token sequence), V plain, SwiGLU on
    the rest.  Sampled tokens x sampled whole heads against the oracle; V and
    H bit for bit equal to the SwiGLU kernel's (the same epilogue there)."""
    import torch
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    from oracle import rope as orope
    from synth import token_positions
    c, p, _ = layers[0]
    n_plain = n_ff = 18432
    n_rope, d_head, axes = 12288, 128, (16, 56, 56)
    perm = gprep.swiglu_row_order(n_plain, n_ff).numpy()
    pw = w4.pack_weight(to_dev_f32(p["R"][perm]))
    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, c.N, c.K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                        to_dev_bf16(p["L2t"][perm]), None)
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    tab = orope.table(orope.angles(token_positions(512, 128, 128), axes, 10000.0))
    assert tab.shape == (c.M, d_head)
    Y0, H0 = w4.gemm_swiglu(qa, w, n_plain)
    Y, H = w4.gemm_rope(qa, w, torch.from_numpy(tab).cuda(), n_rope, d_head, n_plain=n_plain)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    assert torch.equal(H.view(torch.int16), H0.view(torch.int16))
    assert torch.equal(Y[:, n_rope:].view(torch.int16), Y0[:, n_rope:].view(torch.int16))

    g = rng(46)
    rows = np.sort(g.choice(c.M, 64, replace=False))
    rows[0], rows[-1] = 0, c.M - 1                       # a text token and the last image token
    heads = np.sort(g.choice(n_rope // d_head, 6, replace=False))
    heads[-1] = n_rope // d_head - 1
    cols = (heads[:, None] * d_head + np.arange(d_head)[None, :]).reshape(-1)
    oq, osf, ot, _ = nvfp4.quantize(p["R"][cols], amax=np.max(np.abs(p["R"])))
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], nvfp4.pack(oq), osf, ot, p["L1t"], p["L2t"][cols], None,
                                   rows=rows)
    want = orope.rotate(y_ref, tab[rows], len(cols), d_head)
    got = from_dev_bf16(Y[torch.from_numpy(rows).cuda()])[:, cols]
    check_y(got, want)
