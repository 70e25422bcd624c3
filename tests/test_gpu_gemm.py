"""GPU parity of the fused W4A4 GEMM (w4a4_gemm / w4a4_linear) against the
oracle's fp64 product of the dequantised operands plus the fp64 low-rank
branch: relative Frobenius error <= 2e-3 and per-row max |dY| <= 1e-2 of the
row's largest reference value."""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, prepare, to_dev_bf16, to_dev_f32
from oracle import gelu as ogelu
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


def device_weight(w4, p, bias, r):
    """Upload the oracle-packed weight bundle (codes/scales are oracle bytes)."""
    import torch
    N, K = p["R"].shape
    Wq = torch.from_numpy(p["Wq"]).cuda()
    # row-major scales -> SF atoms
    rb = -(-N // 128)
    sfr = np.zeros((rb * 128, K // 16), np.uint8)
    sfr[:N] = p["Wsf"]
    atoms = sfr.reshape(rb, 4, 32, K // 64, 4).transpose(0, 3, 2, 1, 4).reshape(-1)
    Wsf = torch.from_numpy(np.ascontiguousarray(atoms)).cuda()
    t_w = to_dev_f32(np.array([p["t_w"]], np.float32))
    L1t = to_dev_bf16(p["L1t"]) if r else None
    L2t = to_dev_bf16(p["L2t"]) if r else None
    b = to_dev_bf16(bias) if bias is not None else None
    return w4.PackedWeight(Wq, Wsf, t_w, N, K, to_dev_f32(p["inv_s"]), L1t, L2t, b)


def run_case(w4, c, rows=None, epilogue=0, use_linear=True, exact_svd=None):
    import torch
    p = prepare(c, exact_svd=exact_svd)
    if c.r == 0:
        p["L1t"] = None
        p["L2t"] = None
    w = device_weight(w4, p, c.bias, c.r)
    X = to_dev_bf16(c.x)
    if use_linear:
        Y = w4.linear(X, w, epilogue=epilogue)
    else:
        qa = w4.quantize_act(X, w.inv_s, w.L1t, w.t_w)
        Y = w4.gemm(qa, w, epilogue=epilogue)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y = from_dev_bf16(Y)
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], p["Wq"], p["Wsf"], p["t_w"], p["L1t"], p["L2t"],
                                   c.bias, rows=rows)
    if epilogue == 1:
        y_ref = ogelu.gelu_tanh(y_ref)
    return (y if rows is None else y[rows]), y_ref


@pytest.mark.parametrize("M,K,N,r,bias", [
    (128, 256, 192, 32, True),      # one row block: three 128 x 64 tiles (double-buffered accumulator)
    (300, 512, 384, 32, True),      # ragged M, two N tiles
    (300, 512, 264, 32, False),     # 256-wide tiles, ragged N (264 = 256 + 8)
    (257, 768, 576, 0, True),       # no low-rank branch
    (1, 256, 512, 32, True),        # a single token
    (640, 1024, 1024, 32, True),    # several tiles per CTA row
    (300, 512, 384, 16, True),      # rank 16, CTA pairs
    (100, 768, 264, 16, True),      # rank 16, single-CTA kernel, ragged N
    (64, 256, 19200, 32, True),     # single row block, wide: 128 x 192 tiles
    (64, 256, 19456, 0, False),     # single row block, wide: 128 x 256 tiles
])
def test_gemm_small(w4, M, K, N, r, bias):
    c = make_linear("t", M, K, N, r=r, act="normal_outliers", n_out=4, out_scale=100.0,
                    bias_std=0.01 if bias else 0.0, seed=M + K + N)
    y, y_ref = run_case(w4, c)
    check_y(y, y_ref)


def test_gemm_split_entry_points_and_gelu(w4):
    c = make_linear("t", 200, 512, 384, r=32, act="student_t", bias_std=0.01, seed=3)
    y, y_ref = run_case(w4, c, use_linear=False, epilogue=1)
    check_y(y, y_ref)


def test_gemm_exact_operands(w4):
    """Grid-valued operands with a 6 in every block quantise exactly, so Y is
    the exact product rounded once to bf16."""
    import torch
    g = rng(8)
    M, K, N = 256, 512, 384
    grid = np.array(nvfp4.E2M1_VALUES[:8], np.float32)
    x = (grid[g.integers(0, 8, (M, K))] * g.choice([-1, 1], (M, K))).astype(np.float32)
    wv = (grid[g.integers(0, 8, (N, K))] * g.choice([-1, 1], (N, K))).astype(np.float32)
    x[:, ::16] = 6.0
    wv[:, ::16] = -6.0
    wq, wsf, tw, _ = nvfp4.quantize_activation(wv, None)
    p = {"R": wv, "Wq": wq, "Wsf": wsf, "t_w": tw, "inv_s": np.ones(K, np.float32), "L1t": None, "L2t": None}
    w = device_weight(w4, p, None, 0)
    Y = w4.linear(to_dev_bf16(x), w)
    torch.cuda.synchronize()
    y = from_dev_bf16(Y)
    exact = x.astype(np.float64) @ wv.astype(np.float64).T
    # The exact values are multiples of 1/4 below 2^15, so they are exact in
    # fp32.  The GPU value differs from them by a few fp32 ulps (the t_x t_w
    # product is rounded), so one bf16 rounding gives bf16(exact) except where
    # exact sits half-way between two bf16 neighbours; there either neighbour
    # is a correct rounding.
    ex32 = exact.astype(np.float32)
    assert np.array_equal(ex32.astype(np.float64), exact)
    bits = ex32.view(np.uint32)
    tie = (bits & 0xFFFF) == 0x8000
    down = (bits & 0xFFFF0000).view(np.float32).astype(np.float64)
    up = ((bits & 0xFFFF0000) + 0x10000).view(np.float32).astype(np.float64)
    assert np.array_equal(y[~tie], bf16_round(ex32)[~tie].astype(np.float64))
    assert np.all((y[tie] == down[tie]) | (y[tie] == up[tie]))


def test_gemm_config1_full(w4):
    c = config_cases(1)[0]
    y, y_ref = run_case(w4, c)
    check_y(y, y_ref)


def test_gemm_config2_full_sampled_rows(w4):
    c = config_cases(2)[0]
    rows = np.sort(rng(2024).choice(c.M, 384, replace=False))
    rows[-1] = c.M - 1
    y, y_ref = run_case(w4, c, rows=rows)
    check_y(y, y_ref)


def test_empty_batch(w4):
    """An empty batch (M = 0) through the tensor-level API: no-ops with
    empty outputs and a clean device status."""
    import torch
    c = make_linear("t", 1, 512, 256, r=32, act="normal_outliers", seed=4)
    p = prepare(c)
    w = device_weight(w4, p, c.bias, 32)
    X = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    qa = w4.quantize_act(X, w.inv_s, w.L1t, w.t_w)
    Y = w4.gemm(qa, w)
    Z = w4.linear(X, w)
    torch.cuda.synchronize()
    assert tuple(Y.shape) == (0, 256) and tuple(Z.shape) == (0, 256)
    assert w4.w4a4_device_status() == 0
