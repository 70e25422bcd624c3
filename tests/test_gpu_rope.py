"""GPU parity of the rotary-embedding epilogue (w4a4_gemm_rope).

The oracle evaluates the fused projection in fp64 (oracle.linear), turns the
leading query/key features pair by pair by the same fp32 (cos, sin) table the
kernel reads (oracle.rope), and applies SwiGLU to the gate/up features
(oracle.swiglu).  Tables come from the oracle's own angle schedule over the
integer positions of a text + image token sequence.  Two exact checks pin the
kernel's pairing and signs without any tolerance: a table of (1, 0) gives the
SwiGLU kernel's outputs bit for bit, and a table of (0, 1) gives its plain
outputs with every pair (a, b) turned into (-b, a).
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, prepare, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import rope as orope
from oracle import swiglu as oswiglu
from synth import make_linear, rng, token_positions

pytestmark = pytest.mark.gpu

AXES = {32: (8, 12, 12), 64: (16, 24, 24), 128: (16, 56, 56), 256: (32, 112, 112)}


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def positions(M):
    """Text tokens then a near-square grid of image tokens, M in total."""
    side = int(np.sqrt(max(M - 16, 1)))
    n_text = M - side * side
    return token_positions(n_text, side, side)


def build(w4, M, K, n_plain, n_ff, r, seed):
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    N = n_plain + 2 * n_ff
    c = make_linear("qkv_rope", M, K, N, r=r, act="student_t", bias_std=0.5, seed=seed)
    p = prepare(c)
    perm = gprep.swiglu_row_order(n_plain, n_ff).numpy()
    pw = w4.pack_weight(to_dev_f32(p["R"][perm]))
    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, N, K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]) if r else None,
                        to_dev_bf16(p["L2t"][perm]) if r else None, to_dev_bf16(c.bias[perm]))
    qa = w4.quantize_act(to_dev_bf16(c.x), w.inv_s, w.L1t, w.t_w)
    return c, p, w, qa


def device_table(tab, pad):
    import torch
    t = np.zeros((tab.shape[0], tab.shape[1] + pad), np.float32)
    t[:, :tab.shape[1]] = tab
    t[:, tab.shape[1]:] = np.nan          # padding is never read
    return torch.from_numpy(t).cuda()


@pytest.mark.parametrize("M,K,n_plain,n_ff,n_rope,d_head,r,pad", [
    (300, 512, 512, 0, 256, 64, 32, 0),       # ragged rows, no SwiGLU, half the plain features turned
    (300, 512, 512, 384, 512, 128, 32, 8),    # every plain feature turned, SwiGLU, padded table rows
    (128, 768, 256, 128, 256, 32, 16, 4),     # one row block, 32-feature heads, rank 16
    (384, 256, 768, 0, 512, 256, 0, 0),       # 256-feature heads (a whole tile half), no low-rank branch
    (4608, 3072, 768, 768, 512, 128, 32, 0),  # the 1024px sequence: 36 row blocks
])
def test_rope_epilogue(w4, M, K, n_plain, n_ff, n_rope, d_head, r, pad):
    import torch
    c, p, w, qa = build(w4, M, K, n_plain, n_ff, r, seed=M + K + n_rope + d_head)
    tab = orope.table(orope.angles(positions(M), AXES[d_head], 10000.0))
    s_next = (1.0 / np.exp(0.3 * rng(9).standard_normal(max(n_ff, 1)))).astype(np.float32)
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    Y, H = w4.gemm_rope(qa, w, device_table(tab, pad), n_rope, d_head, n_plain=n_plain,
                        next_inv_s=to_dev_f32(s_next) if n_ff else None, next_amax=amax if n_ff else None)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"], c.bias)
    plain_ref, h_ref = oswiglu.split_fused(y_ref, n_plain, n_ff)
    y = from_dev_bf16(Y)
    want = orope.rotate(plain_ref, tab, n_rope, d_head)
    check_y(y[:, :n_rope], want[:, :n_rope])
    if n_rope < n_plain:
        check_y(y[:, n_rope:], want[:, n_rope:])
    if n_ff:
        h = from_dev_bf16(H)
        check_y(h, h_ref)
        xs = (h * s_next[None, :]).astype(np.float32)
        assert float(amax.cpu()[0]) == float(np.max(np.abs(xs)))
    else:
        assert H is None


@pytest.mark.parametrize("n_ff", [0, 256])
def test_rope_exact_turns(w4, n_ff):
    """(cos, sin) = (1, 0): the SwiGLU kernel's outputs, bit for bit;
    (0, 1): its plain outputs with each pair (a, b) -> (-b, a), bit for bit."""
    import torch
    M, K, n_plain, n_rope, d_head = 520, 512, 768, 512, 128
    c, p, w, qa = build(w4, M, K, n_plain, n_ff, 32, seed=77 + n_ff)
    if n_ff:
        Y0, H0 = w4.gemm_swiglu(qa, w, n_plain)
    else:
        Y0, H0 = w4.gemm(qa, w), None
    ident = torch.zeros(M, d_head, dtype=torch.float32, device="cuda")
    ident[:, 0::2] = 1.0
    Y1, H1 = w4.gemm_rope(qa, w, ident, n_rope, d_head, n_plain=n_plain)
    quarter = torch.zeros(M, d_head, dtype=torch.float32, device="cuda")
    quarter[:, 1::2] = 1.0
    Y2, H2 = w4.gemm_rope(qa, w, quarter, n_rope, d_head, n_plain=n_plain)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    assert torch.equal(Y1.view(torch.int16), Y0.view(torch.int16))
    if n_ff:
        assert torch.equal(H1.view(torch.int16), H0.view(torch.int16))
        assert torch.equal(H2.view(torch.int16), H0.view(torch.int16))
    turned = Y0[:, :n_rope].clone()
    turned[:, 0::2] = -Y0[:, 1:n_rope:2]
    turned[:, 1::2] = Y0[:, 0:n_rope:2]
    assert torch.equal(Y2[:, :n_rope].view(torch.int16), turned.view(torch.int16))
    assert torch.equal(Y2[:, n_rope:].view(torch.int16), Y0[:, n_rope:].view(torch.int16))


def test_rope_table_builder_matches_the_oracle(w4):
    """prep.rope_table (torch, on the GPU) against the oracle's table: the same
    fp64 angles rounded once to fp32, so at most one fp32 ulp apart."""
    import torch
    from bit_diffusion_transformer_nvfp4_b200 import prep as gprep
    pos = token_positions(512, 128, 128)
    got = gprep.rope_table(torch.from_numpy(pos).cuda(), AXES[128]).cpu().numpy()
    want = orope.table(orope.angles(pos, AXES[128], 10000.0))
    assert got.shape == want.shape
    np.testing.assert_allclose(got, want, rtol=0, atol=2 ** -24)
