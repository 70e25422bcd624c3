"""GPU parity of the NVFP4 quantiser (nvfp4_quantize_act, nvfp4_pack_weight)
against the oracle: codes, scale bytes and the tensor scale bit for bit; the
low-rank U within fp32 rounding."""
import numpy as np
import pytest

from helpers import prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4
from synth import bf16_round, config_cases, make_linear, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def run_quant(w4, x, inv_s=None, L1t=None, t_w=None):
    import torch
    M, K = x.shape
    X = to_dev_bf16(x)
    qa = w4.quantize_act(X, None if inv_s is None else to_dev_f32(inv_s),
                         None if L1t is None else to_dev_bf16(L1t),
                         None if t_w is None else to_dev_f32(np.array([t_w], np.float32)))
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    sf = sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K)
    return qa, qa.Xq.cpu().numpy(), sf, float(qa.t_x.cpu().numpy()[0])


def check_bytes(x, inv_s, xq, sf, t):
    M, K = x.shape
    oq, osf, ot, _ = nvfp4.quantize_activation(x, inv_s)
    assert t == float(ot), (t, float(ot))
    np.testing.assert_array_equal(sf[:M], osf)
    assert not sf[M:].any(), "pad rows of the scale atoms must be zero"
    bad = np.argwhere(xq != oq)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:5].tolist()}: gpu {xq[tuple(bad[0])]:#x} oracle {oq[tuple(bad[0])]:#x}"


def edge_matrix():
    """Rows exercising the quantiser's special cases (all values bf16-exact)."""
    K = 512
    g = rng(77)
    x = np.zeros((12, K), np.float32)
    x[1] = g.standard_normal(K); x[1, 100] = 3.0e4                 # one huge outlier (the tensor max)
    x[2] = g.standard_normal(K) * 1e-6                               # blocks whose scale underflows
    x[3, :16] = [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]
    x[3, 16:32] = x[3, :16] / 64
    x[4] = 6.0 * 2.0 ** g.integers(-8, 8, K)                         # rows of 6 * 2^k
    x[5] = -np.abs(g.standard_normal(K)) * 1e-3                      # small negatives -> -0 codes
    x[6, ::2] = -0.0
    x[7] = g.standard_normal(K) * 448.0
    x[8] = np.repeat(g.standard_normal(K // 16), 16)                 # constant blocks
    x[9] = g.standard_normal(K) * np.exp(3 * g.standard_normal(K))
    x[10] = np.float32(2.0 ** -100)                                  # tiny but normal
    x[11] = g.standard_normal(K)
    return bf16_round(x)


def test_quant_edge_cases(w4):
    x = edge_matrix()
    qa, xq, sf, t = run_quant(w4, x)
    check_bytes(x, None, xq, sf, t)


def test_quant_all_zero(w4):
    x = np.zeros((64, 256), np.float32)
    qa, xq, sf, t = run_quant(w4, x)
    assert t == 1.0 and not xq.any() and not sf.any()


@pytest.mark.parametrize("M,K", [(1, 256), (127, 256), (128, 512), (300, 512), (257, 1024), (1000, 768)])
def test_quant_shapes_with_smoothing(w4, M, K):
    g = rng(M * 7 + K)
    x, _ = (g.standard_normal((M, K)).astype(np.float32), None)
    x[:, g.choice(K, 5, replace=False)] *= 80
    x = bf16_round(x)
    inv_s = (1.0 / np.exp(0.5 * g.standard_normal(K))).astype(np.float32)
    qa, xq, sf, t = run_quant(w4, x, inv_s)
    check_bytes(x, inv_s, xq, sf, t)


@pytest.mark.parametrize("M,K,r,given", [
    (300, 512, 32, False),     # single pass
    (300, 512, 16, False),     # single pass, rank 16
    (300, 512, 16, True),      # streaming pass with the amax given, rank 16
    (2048, 12288, 16, False),  # two passes (the tile set is not co-resident), rank 16
])
def test_quant_lowrank_u(w4, M, K, r, given):
    import torch
    c = make_linear("t", M, K, 384, r=r, act="normal_outliers", n_out=6, out_scale=100.0, seed=5 + r)
    p = prepare(c)
    if given:
        a = np.max(np.abs((c.x * p["inv_s"][None, :]).astype(np.float32)))
        qa = w4.quantize_act(to_dev_bf16(c.x), to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                             to_dev_f32(np.array([p["t_w"]], np.float32)), amax=to_dev_f32(np.array([a], np.float32)))
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0
        xq, sf, t = qa.Xq.cpu().numpy(), sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K), float(qa.t_x.cpu()[0])
    else:
        qa, xq, sf, t = run_quant(w4, c.x, p["inv_s"], p["L1t"], float(p["t_w"]))
    check_bytes(c.x, p["inv_s"], xq, sf, t)
    assert tuple(qa.U.shape) == (M, 2 * r)
    U = qa.U.float().cpu().numpy()
    hi, lo = U[:, :r], U[:, r:]
    alpha = np.float64(np.float32(np.float32(t) * np.float32(p["t_w"])))
    ref = olinear.lowrank_down(c.x, p["L1t"]) / alpha
    got = hi.astype(np.float64) + lo.astype(np.float64)
    # fp32 accumulation of K exact bf16 products (about sqrt(K) * 2^-24
    # relative, 1.4e-6 at K = 512) plus the hi|lo representation (2^-17)
    assert olinear.rel_frobenius(got, ref) < 1e-5
    assert np.max(np.abs(got - ref)) <= 5e-5 * np.max(np.abs(ref))
    # hi holds the leading bf16 part: |lo| is at most half a bf16 ulp of hi
    # (plus lo's own rounding)
    assert np.all(np.abs(lo) <= np.abs(hi) * 2.0 ** -8 * (1 + 2.0 ** -7))


def test_sf_to_rowmajor_entry(w4):
    """The C-ABI layout helper equals the test's own numpy rearrangement of
    the SF atoms, on activation scales (ragged rows) and weight scales."""
    import torch
    g = rng(77)
    x = bf16_round(g.standard_normal((300, 768)).astype(np.float32) * 3.0)
    qa = w4.quantize_act(to_dev_bf16(x))
    got = w4.sf_rowmajor(qa.Xsf, 300, 768)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy(), sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), 300, 768)[:300])
    pw = w4.pack_weight(to_dev_f32(g.standard_normal((520, 512)).astype(np.float32)))
    got = w4.sf_rowmajor(pw.Wsf, 520, 512)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(got.cpu().numpy(), sf_atoms_to_rowmajor(pw.Wsf.cpu().numpy(), 520, 512)[:520])


@pytest.mark.parametrize("cfg", [1, 2])
def test_quant_config_full_size(w4, cfg):
    c = config_cases(cfg)[0]
    g = rng(cfg)
    inv_s = (1.0 / np.exp(0.3 * g.standard_normal(c.K))).astype(np.float32)
    qa, xq, sf, t = run_quant(w4, c.x, inv_s)
    check_bytes(c.x, inv_s, xq, sf, t)


@pytest.mark.parametrize("src", ["f32", "bf16"])
def test_pack_weight(w4, src):
    import torch
    c = make_linear("w", 16, 768, 520, r=32, act="normal_outliers", seed=9)
    p = prepare(c)
    R = p["R"] if src == "f32" else bf16_round(p["R"])
    Rd = to_dev_f32(R) if src == "f32" else to_dev_bf16(R)
    pw = w4.pack_weight(Rd)
    torch.cuda.synchronize()
    wq = pw.Wq.cpu().numpy()
    wsf = sf_atoms_to_rowmajor(pw.Wsf.cpu().numpy(), c.N, c.K)
    oq, osf, ot, _ = nvfp4.quantize_activation(R, None)
    assert float(pw.t_w.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(wsf[:c.N], osf)
    np.testing.assert_array_equal(wq, oq)


@pytest.mark.parametrize("M,K", [(4608, 3072), (1024, 12288)])
def test_quant_lowrank_stage_reuse(w4, M, K):
    """Enough K per CTA that the TMA ring stages are refilled while the
    low-rank MMAs also read them: codes bit-exact and identical run to run."""
    import torch
    c = make_linear("t", M, K, 256, r=32, act="normal_outliers", n_out=8, out_scale=60.0, seed=M + K)
    p = prepare(c)
    X = to_dev_bf16(c.x)
    args = (to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]), to_dev_f32(np.array([p["t_w"]], np.float32)))
    qa = w4.quantize_act(X, *args)
    qb = w4.quantize_act(X, *args)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    assert torch.equal(qa.Xq, qb.Xq) and torch.equal(qa.Xsf, qb.Xsf) and torch.equal(qa.U, qb.U)
    check_bytes(c.x, p["inv_s"], qa.Xq.cpu().numpy(), sf_atoms_to_rowmajor(qa.Xsf.cpu().numpy(), M, K),
                float(qa.t_x.cpu()[0]))


def test_quant_two_pass_full_size(w4):
    """The 12288-deep MLP down-projection input (4608 x 12288) needs more K
    slices than can be co-resident, so it takes the two-pass quantiser
    (column-maxima amax pass, then the grouped quantise pass with the U MMAs
    and the cross-slice U sums): every code and scale byte bit for bit, U on
    sampled rows within fp32 rounding."""
    c = config_cases(3)[1]
    g = rng(33)
    inv_s = (1.0 / np.exp(0.3 * g.standard_normal(c.K))).astype(np.float32)
    L1t = bf16_round((g.standard_normal((32, c.K)) * 0.02).astype(np.float32))
    t_w = 0.01
    qa, xq, sf, t = run_quant(w4, c.x, inv_s, L1t, t_w)
    check_bytes(c.x, inv_s, xq, sf, t)
    rows = np.sort(g.choice(c.M, 256, replace=False))
    rows[-1] = c.M - 1
    U = qa.U.float().cpu().numpy()[rows]
    got = U[:, :32].astype(np.float64) + U[:, 32:].astype(np.float64)
    alpha = np.float64(np.float32(np.float32(t) * np.float32(t_w)))
    ref = olinear.lowrank_down(c.x[rows], L1t) / alpha  # U uses the raw X and L1t as given
    assert olinear.rel_frobenius(got, ref) < 1e-5
