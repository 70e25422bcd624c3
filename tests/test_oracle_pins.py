"""Pins for the oracle: each check ties it to something other than itself.

Sources of truth used here: hand-written tables of the number formats, the
hand-worked byte example under tests/golden/, exact invariants of the
quantiser (power-of-two scaling, idempotence), a scalar brute-force
restatement for tiny inputs, library routines for special cases (LAPACK SVD,
torch's GELU), and algebraic identities of the SVDQuant decomposition.
"""
import os
import struct

import numpy as np
import pytest

from oracle import gelu, linear, nvfp4, prep
from synth import bf16_round, rng

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(v):
    return float(np.float32(v))


# ---------------------------------------------------------------- formats

def test_e2m1_table_by_hand():
    want = [0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6]
    got = nvfp4.E2M1_VALUES
    assert list(got) == want
    assert np.signbit(got[8])          # code 0x8 is -0


def test_e2m1_every_code_round_trips():
    for c in range(16):
        assert int(nvfp4.e2m1_encode(np.float32(nvfp4.E2M1_VALUES[c]))) == c


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),  # ties -> even
    (np.nextafter(np.float32(0.25), np.float32(1)), 1),
    (np.nextafter(np.float32(5.0), np.float32(0)), 6),
    (np.nextafter(np.float32(5.0), np.float32(9)), 7),
    (6.0, 7), (6.5, 7), (1e30, 7),                                              # satfinite
    (0.1, 0), (-0.1, 8), (-0.0, 8), (-0.3, 9), (-5.0, 14), (-100.0, 15),
])
def test_e2m1_rounding_by_hand(v, code):
    assert int(nvfp4.e2m1_encode(np.float32(v))) == code


def test_e4m3_decode_by_hand():
    d = nvfp4.e4m3_decode
    assert d(0x38) == 1.0
    assert d(0x7E) == 448.0                       # largest finite, the +-448 range
    assert d(0x01) == 2.0 ** -9                   # smallest subnormal
    assert d(0x07) == 7 * 2.0 ** -9
    assert d(0x08) == 2.0 ** -6                   # smallest normal
    assert d(0x4E) == 7.0                         # 1.75 * 2^2
    assert d(0x00) == 0.0
    assert np.isnan(d(0x7F))


def test_e4m3_every_finite_byte_round_trips():
    for b in range(127):
        assert int(nvfp4.e4m3_encode_nonneg(np.float32(nvfp4.E4M3_VALUES[b]))) == b


@pytest.mark.parametrize("v,byte", [
    (1.0625, 0x38), (1.1875, 0x3A),                 # ties between 1,1.125 and 1.125,1.25
    (2.0 ** -10, 0x00), (3 * 2.0 ** -10, 0x02),      # subnormal ties
    (449.0, 0x7E), (464.0, 0x7E), (1e6, 0x7E),       # saturation
    (0.0, 0x00), (2.0 ** -12, 0x00),
])
def test_e4m3_rounding_by_hand(v, byte):
    assert int(nvfp4.e4m3_encode_nonneg(np.float32(v))) == byte


# ---------------------------------------------------------------- hand-packed example

def _golden():
    out = {}
    with open(os.path.join(GOLDEN, "nvfp4_handpacked.txt")) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


def test_handpacked_bytes():
    g = _golden()
    b0 = np.array([float(v) for v in g["input_block0"]], np.float32)
    b1 = (b0 / np.float32(float(g["input_block1_divisor"][0]))).astype(np.float32)
    x = np.concatenate([b0, b1])[None, :]
    packed, sf, t, amax = nvfp4.quantize_activation(x, None)
    assert amax == 6.0
    assert list(packed[0, :8]) == [int(h, 16) for h in g["packed_block0_hex"]]
    assert list(packed[0, 8:]) == [int(h, 16) for h in g["packed_block1_hex"]]
    assert list(sf[0]) == [int(h, 16) for h in g["scale_bytes_hex"]]
    codes, _, _, _ = nvfp4.quantize(x)
    assert list(codes[0, :16]) == [int(c) for c in g["codes_block0"]]


# ---------------------------------------------------------------- scalar brute force

def _e2m1_brute(v):
    grid = [0, .5, 1, 1.5, 2, 3, 4, 6]
    a = abs(v)
    best = None
    for i, gv in enumerate(grid):
        d = abs(a - gv)
        if best is None or d < best[0] or (d == best[0] and i % 2 == 0):
            best = (d, i)
    i = 7 if a >= 6 else best[1]
    neg = struct.unpack("<I", struct.pack("<f", v))[0] >> 31
    return i | (neg << 3)


def _e4m3_brute(v):
    best = None
    for b in range(127):
        gv = nvfp4.e4m3_decode_byte(b)
        d = abs(v - gv)
        if best is None or d < best[0] or (d == best[0] and b % 2 == 0):
            best = (d, b)
    return 0x7E if v >= 448 else best[1]


def _quantize_brute(rows):
    """Element-by-element restatement of the quantiser with Python loops."""
    amax = 0.0
    for row in rows:
        for v in row:
            amax = max(amax, abs(v))
    t = f32(f32(amax) / f32(2688.0))
    if not (t >= 2.0 ** -126):
        t = 1.0
    rt = f32(1.0 / t)
    codes, sfs = [], []
    for row in rows:
        crow, srow = [], []
        for k0 in range(0, len(row), 16):
            blk = row[k0:k0 + 16]
            b = max(abs(v) for v in blk)
            e = _e4m3_brute(f32(f32(b * rt) / 6.0))
            sd = nvfp4.e4m3_decode_byte(e)
            srow.append(e)
            if sd == 0:
                crow += [0] * 16
            else:
                rq = f32(1.0 / f32(sd * t))
                crow += [_e2m1_brute(f32(v * rq)) for v in blk]
        codes.append(crow)
        sfs.append(srow)
    return np.array(codes, np.uint8), np.array(sfs, np.uint8), np.float32(t)


@pytest.mark.parametrize("seed", range(6))
def test_quantiser_matches_scalar_brute_force(seed):
    g = rng(seed)
    rows, K = 3, 64
    x = g.standard_normal((rows, K)).astype(np.float32) * np.float32(10.0 ** g.uniform(-6, 3))
    x[0, 5] *= 300.0                        # an outlier
    x[1, 16:32] *= 1e-7                     # a block that underflows to scale 0
    x[2, 0] = -0.0
    x = x.astype(np.float32)
    c_ref, s_ref, t_ref = _quantize_brute(x.tolist())
    c, s, t, _ = nvfp4.quantize(x)
    assert t == t_ref
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(c, c_ref)


# ---------------------------------------------------------------- invariants

def test_power_of_two_scaling_invariance():
    g = rng(11)
    x = bf16_round(g.standard_normal((8, 256)).astype(np.float32) * 3)
    c0, s0, t0, _ = nvfp4.quantize(x)
    for j in (-20, -7, -1, 1, 5, 20):
        c, s, t, _ = nvfp4.quantize((x * np.float32(2.0 ** j)).astype(np.float32))
        np.testing.assert_array_equal(c, c0)
        np.testing.assert_array_equal(s, s0)
        assert t == np.float32(t0 * np.float32(2.0 ** j))


def test_idempotent():
    g = rng(12)
    x = (g.standard_normal((16, 512)) * np.exp(2 * g.standard_normal(512))).astype(np.float32)
    c, s, t, _ = nvfp4.quantize(x)
    d = nvfp4.dequantize(c, s, t).astype(np.float32)
    c2, s2, _, _ = nvfp4.quantize(d)
    np.testing.assert_array_equal(s2, s)
    # -0 codes dequantise to -0.0 and re-encode to 0x8; +0 stays 0x0
    np.testing.assert_array_equal(c2, c)


def test_largest_block_takes_largest_scale_and_error_bound():
    g = rng(13)
    x = (g.standard_normal((32, 1024)) * np.exp(g.standard_normal(1024))).astype(np.float32)
    c, s, t, amax = nvfp4.quantize(x)
    i, k = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert s[i, k // 16] == 0x7E
    sd = nvfp4.e4m3_decode(s).astype(np.float64)
    err = np.abs(x.astype(np.float64) - nvfp4.dequantize(c, s, t)).reshape(32, 64, 16)
    unit = (sd * float(t))[:, :, None]
    ok = sd[:, :, None] > 0
    # worst rounding step of the E2M1 grid is 1 (between 4 and 6); saturation of
    # the block maximum adds at most 6/(1-1/16) - 6 = 0.4 < 1
    assert np.all(err[np.broadcast_to(ok, err.shape)] <= 1.0 * np.broadcast_to(unit, err.shape)[np.broadcast_to(ok, err.shape)] * (1 + 1e-6))


def test_row_subset_under_whole_tensor_scale():
    """Once the tensor scale is fixed each row quantises on its own: a subset
    of rows under the whole tensor's amax gives exactly those rows' bytes."""
    g = rng(15)
    x = bf16_round((g.standard_normal((40, 256)) * np.exp(g.standard_normal(256))).astype(np.float32))
    inv_s = (1.0 / np.exp(0.2 * g.standard_normal(256))).astype(np.float32)
    q, s, t, a = nvfp4.quantize_activation(x, inv_s)
    rows = np.array([0, 7, 8, 39])
    q2, s2, t2, a2 = nvfp4.quantize_activation(x, inv_s, rows)
    assert t2 == t and a2 == a
    np.testing.assert_array_equal(q2, q[rows])
    np.testing.assert_array_equal(s2, s[rows])


def test_all_zero_tensor():
    c, s, t, amax = nvfp4.quantize(np.zeros((4, 64), np.float32))
    assert amax == 0 and t == 1.0
    assert not c.any() and not s.any()


def test_pack_unpack():
    g = rng(14)
    c = g.integers(0, 16, size=(5, 64)).astype(np.uint8)
    p = nvfp4.pack(c)
    assert p.shape == (5, 32)
    assert p[0, 0] == (c[0, 0] | (c[0, 1] << 4))
    np.testing.assert_array_equal(nvfp4.unpack(p), c)


# ---------------------------------------------------------------- linear + prep

def test_linear_matches_triple_loop():
    g = rng(21)
    M, K, N, r = 3, 32, 5, 2
    x = bf16_round(g.standard_normal((M, K)).astype(np.float32))
    inv_s = (1.0 / np.exp(0.3 * g.standard_normal(K))).astype(np.float32)
    R = (0.05 * g.standard_normal((N, K))).astype(np.float32)
    L1t = bf16_round(g.standard_normal((r, K)).astype(np.float32) * 0.1)
    L2t = bf16_round(g.standard_normal((N, r)).astype(np.float32) * 0.1)
    bias = bf16_round(g.standard_normal(N).astype(np.float32) * 0.01)
    wq, wsf, tw, _ = nvfp4.quantize_activation(R, None)
    y, aux = linear.w4a4_linear(x, inv_s, wq, wsf, tw, L1t, L2t, bias)
    xc, xs, tx = aux["xq"], aux["xsf"], aux["t_x"]
    xcodes, wcodes = nvfp4.unpack(xc), nvfp4.unpack(wq)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += (nvfp4.e2m1_decode_code(int(xcodes[m, k])) * nvfp4.e4m3_decode_byte(int(xs[m, k // 16])) * float(tx)
                        * nvfp4.e2m1_decode_code(int(wcodes[n, k])) * nvfp4.e4m3_decode_byte(int(wsf[n, k // 16])) * float(tw))
            for j in range(r):
                u = sum(float(x[m, k]) * float(L1t[j, k]) for k in range(K))
                acc += u * float(L2t[n, j])
            acc += float(bias[n])
            assert abs(acc - y[m, n]) <= 1e-12 * max(1.0, abs(acc))


def test_full_rank_decomposition_reproduces_dense_product():
    """r = min(N, K): the low-rank branch is the whole smoothed weight, the
    residual is zero, and the layer is X W^T + b up to bf16 rounding of L1/L2."""
    g = rng(22)
    M, K, N = 8, 32, 16
    x = bf16_round(g.standard_normal((M, K)).astype(np.float32))
    x[:, 3] *= 50
    x = bf16_round(x)
    w = bf16_round((0.02 * g.standard_normal((N, K))).astype(np.float32))
    b = bf16_round((0.01 * g.standard_normal(N)).astype(np.float32))
    p = prep.svdquant_prepare(w, x, r=min(N, K))
    assert np.abs(p["R"]).max() < 1e-6 * np.abs(w).max() * 100
    wq, wsf, tw, _ = nvfp4.quantize_activation(p["R"], None)
    y, _ = linear.w4a4_linear(x, p["inv_s"], wq, wsf, tw, p["L1t"], p["L2t"], b)
    dense = x.astype(np.float64) @ w.astype(np.float64).T + b
    assert linear.rel_frobenius(y, dense) < 1e-2


def test_rank_zero_with_exact_operands_is_plain_gemm():
    """Operands on the E2M1 grid whose every 16-block holds a 6 quantise to
    themselves (every block scale is 448, the tensor scale 6/2688), so with r=0
    and no smoothing the layer is the exact product."""
    g = rng(23)
    M, K, N = 4, 64, 6
    grid = np.array(nvfp4.E2M1_VALUES[:8], np.float32)
    xv = (grid[g.integers(0, 8, (M, K))] * g.choice([-1, 1], (M, K))).astype(np.float32)
    wv = (grid[g.integers(0, 8, (N, K))] * g.choice([-1, 1], (N, K))).astype(np.float32)
    xv[:, ::16] = 6.0
    wv[:, ::16] = -6.0
    wq, wsf, tw, _ = nvfp4.quantize_activation(wv, None)
    y, _ = linear.w4a4_linear(xv, None, wq, wsf, tw, None, None, None)
    np.testing.assert_allclose(y, xv.astype(np.float64) @ wv.astype(np.float64).T, rtol=1e-6, atol=1e-6)


def test_smoothing_factor_closed_form():
    x_cal = np.array([[4.0, -1.0, 0.0], [-2.0, 0.5, 0.0]])
    w = np.array([[1.0, 4.0, 1.0], [-0.5, 1.0, 2.0]])
    s = prep.smoothing_factors(x_cal, w, alpha=0.5)
    np.testing.assert_allclose(s, [2.0, 0.5, 1.0])


def test_svd_residual_is_eckart_young():
    g = rng(24)
    w = g.standard_normal((40, 64))
    x_cal = g.standard_normal((16, 64))
    r = 5
    p = prep.svdquant_prepare(w, x_cal, r=r, exact_svd=True)
    sv = np.linalg.svd(w * p["s"][None, :], compute_uv=False)
    np.testing.assert_allclose(np.linalg.norm(p["R"].astype(np.float64)) ** 2, (sv[r:] ** 2).sum(), rtol=1e-5)
    pr = prep.svdquant_prepare(w, x_cal, r=r, exact_svd=False)
    np.testing.assert_allclose(np.linalg.norm(pr["R"].astype(np.float64)) ** 2, (sv[r:] ** 2).sum(), rtol=1e-3)


def test_gelu_against_library():
    torch = pytest.importorskip("torch")
    x = np.linspace(-8, 8, 1001)
    ref = torch.nn.functional.gelu(torch.tensor(x, dtype=torch.float64), approximate="tanh").numpy()
    np.testing.assert_allclose(gelu.gelu_tanh(x), ref, rtol=1e-14, atol=1e-15)
    assert gelu.gelu_tanh(np.array([0.0]))[0] == 0.0


def test_bf16_rounding_against_library():
    torch = pytest.importorskip("torch")
    g = rng(25)
    v = (g.standard_normal(10000) * np.exp(4 * g.standard_normal(10000))).astype(np.float32)
    ref = torch.tensor(v).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(prep.to_bf16_values(v), ref)
    np.testing.assert_array_equal(bf16_round(v), ref)


# ---------------------------------------------------------------- parity checkers
# Every Y verdict rests on these two functions, so each is pinned to values
# worked out by hand, on cases where the plausible mistakes (normalising by
# the tested result instead of the reference, reducing over columns or over
# the whole matrix instead of per row) give a different number.

def test_rel_frobenius_by_hand():
    ref = np.array([[1.0, 10.0], [6.0, 8.0]])
    test = np.array([[1.0, 10.0], [6.0, 4.0]])
    # |test - ref|_F = 4, |ref|_F = sqrt(1 + 100 + 36 + 64) = sqrt(201)
    assert linear.rel_frobenius(test, ref) == pytest.approx(4.0 / np.sqrt(201.0), rel=1e-15)
    # normalising by |test|_F = sqrt(153) would give 0.3234 instead of 0.2821
    assert abs(linear.rel_frobenius(test, ref) - 4.0 / np.sqrt(153.0)) > 0.04
    # a 3-4-5 case: the difference (0.3, 0.4) against (3, 4) is exactly 0.1
    assert linear.rel_frobenius(np.array([[3.3, 4.4]]), np.array([[3.0, 4.0]])) == pytest.approx(0.1, rel=1e-12)
    assert linear.rel_frobenius(ref, ref) == 0.0
    # an all-zero reference falls back to the absolute norm of the difference
    assert linear.rel_frobenius(np.array([[0.0, 3.0], [4.0, 0.0]]), np.zeros((2, 2))) == 5.0


def test_row_maxabs_ratio_by_hand():
    ref = np.array([[1.0, 10.0], [6.0, 8.0]])
    test = np.array([[1.0, 10.0], [6.0, 4.0]])
    # row 0: 0 / 10; row 1: |4 - 8| / max(6, 8) = 0.5
    assert linear.row_maxabs_ratio(test, ref) == 0.5
    # over columns it would be 0.4 (4 / 10), over the whole matrix 0.4, and
    # against the tested row's maximum 4 / 6
    assert linear.row_maxabs_ratio(test.T, ref.T) == 0.4
    # a zero reference row is compared in absolute terms
    assert linear.row_maxabs_ratio(np.array([[0.0, 1e-3], [2.0, 2.0]]),
                                   np.array([[0.0, 0.0], [2.0, 2.0]])) == 1e-3
    # the largest row ratio wins, whatever the row order
    a = np.array([[10.0, 0.0], [1.0, 0.0], [4.0, 4.0]])
    b = a + np.array([[1.0, 0.0], [0.5, 0.0], [0.0, -1.0]])
    assert linear.row_maxabs_ratio(b, a) == 0.5
    assert linear.row_maxabs_ratio(b[::-1], a[::-1]) == 0.5


# ---------------------------------------------------------------- SwiGLU

def test_silu_closed_forms():
    from oracle import swiglu
    assert swiglu.silu(np.array([0.0]))[0] == 0.0
    # sigmoid(ln 3) = 3/4, sigmoid(-ln 3) = 1/4
    ln3 = np.log(3.0)
    np.testing.assert_allclose(swiglu.silu(np.array([ln3, -ln3])), [0.75 * ln3, -0.25 * ln3], rtol=1e-15)
    # silu(x) - silu(-x) = x (sigmoid(x) + sigmoid(-x) = 1), for any x
    x = np.linspace(-30, 30, 601)
    np.testing.assert_allclose(swiglu.silu(x) - swiglu.silu(-x), x, rtol=1e-14, atol=1e-14)
    # limits: x for large x, 0 (from below) for very negative x, no overflow warning
    assert swiglu.silu(np.array([800.0]))[0] == 800.0
    v = swiglu.silu(np.array([-800.0]))[0]
    assert v == 0.0 and np.signbit(v)


def test_silu_against_library():
    torch = pytest.importorskip("torch")
    from oracle import swiglu
    x = np.linspace(-20, 20, 2001)
    ref = torch.nn.functional.silu(torch.tensor(x, dtype=torch.float64)).numpy()
    np.testing.assert_allclose(swiglu.silu(x), ref, rtol=1e-15, atol=1e-300)


def test_swiglu_split_by_hand():
    from oracle import swiglu
    # plain 2 columns, then gate (2) and up (2)
    y = np.array([[1.0, 2.0, 0.0, np.log(3.0), 5.0, 4.0]])
    plain, h = swiglu.split_fused(y, 2, 2)
    np.testing.assert_array_equal(plain, [[1.0, 2.0]])
    # silu(0) * 5 = 0; silu(ln 3) * 4 = 0.75 ln 3 * 4 = 3 ln 3
    np.testing.assert_allclose(h, [[0.0, 3.0 * np.log(3.0)]], rtol=1e-15)
    # gate and up are not interchangeable
    _, h2 = swiglu.split_fused(y[:, [0, 1, 4, 5, 2, 3]], 2, 2)
    assert not np.allclose(h, h2)


# ---------------------------------------------------------------- given tensor scale

def test_given_tensor_scale_matches_the_measured_one():
    g = rng(31)
    x = bf16_round(g.standard_normal((40, 128)).astype(np.float32) * 3.0)
    a = np.float32(np.max(np.abs(x)))
    c1, s1, t1, _ = nvfp4.quantize(x, amax=a)
    c2, s2, t2, _ = nvfp4.quantize(x, t=nvfp4.tensor_scale(a))
    assert t1 == t2
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)


def test_given_tensor_scale_by_hand():
    # one block [6, -3, 0.5, 0, ...]: with t = 1 its scale is E4M3(6 / 6) =
    # 1.0 = 0x38 and the codes are the values themselves (6 -> 0x7, -3 -> 0xD,
    # 0.5 -> 0x1); with t = 2 the scale is E4M3(6 * 0.5 / 6) = 0.5 = 0x30 and
    # the codes again the values (x / (0.5 * 2)); with t = 1/128 the block
    # needs 6 * 128 / 6 = 128 -> 0x70 (1.0 * 2^7)
    x = np.zeros((1, 16), np.float32)
    x[0, :3] = [6.0, -3.0, 0.5]
    for t, sbyte in [(1.0, 0x38), (2.0, 0x30), (1.0 / 128, 0x70)]:
        c, sf, tt, _ = nvfp4.quantize(x, t=t)
        assert float(tt) == t and sf[0, 0] == sbyte, (t, hex(sf[0, 0]))
        assert list(c[0, :4]) == [0x7, 0xD, 0x1, 0x0]
    # a scale too small for the data saturates the block scale at 448 and the
    # codes at 6: t = 1/1024 asks for 6 * 1024 / 6 = 1024 > 448
    c, sf, _, _ = nvfp4.quantize(x, t=1.0 / 1024)
    assert sf[0, 0] == 0x7E
    assert c[0, 0] == 0x7
    with pytest.raises(ValueError):
        nvfp4.quantize(x, t=0.0)


# ---------------------------------------------------------------- rotary embedding

def test_rope_rotation_by_hand():
    from oracle import rope
    # one head of 4 features (pairs (0,1) and (2,3)) then two plain columns;
    # pair 0 turned by a quarter turn, pair 1 by a half turn
    y = np.array([[1.0, 0.0, 0.0, 1.0, 3.0, 4.0]])
    tab = rope.table(np.array([[np.pi / 2, np.pi]]))
    got = rope.rotate(y, tab, n_rope=4, d_head=4)
    np.testing.assert_allclose(got, [[0.0, 1.0, 0.0, -1.0, 3.0, 4.0]], atol=1e-7)
    # a sixth of a turn on (2, 0): (2 cos, 2 sin) = (1, sqrt 3); the pairs are
    # adjacent features, not the two halves of the head
    got = rope.rotate(np.array([[2.0, 0.0, 0.0, 0.0]]), rope.table(np.array([[np.pi / 3, 0.0]])), 4, 4)
    np.testing.assert_allclose(got, [[1.0, np.sqrt(3.0), 0.0, 0.0]], atol=1e-7)


def test_rope_every_head_uses_the_same_pairs():
    from oracle import rope
    g = rng(41)
    y = g.standard_normal((3, 24))
    tab = rope.table(g.uniform(-np.pi, np.pi, (3, 4)))
    got = rope.rotate(y, tab, n_rope=16, d_head=8)
    for h0 in (0, 8):
        np.testing.assert_allclose(got[:, h0:h0 + 8], rope.rotate(y[:, h0:h0 + 8], tab, 8, 8), rtol=0, atol=0)
    np.testing.assert_array_equal(got[:, 16:], y[:, 16:])        # past n_rope: unchanged


def test_rope_preserves_pair_norms_and_inverts():
    from oracle import rope
    g = rng(42)
    y = g.standard_normal((5, 32))
    th = g.uniform(-10, 10, (5, 8))
    got = rope.rotate(y, rope.table(th), 32, 16)
    np.testing.assert_allclose(got[:, 0::2] ** 2 + got[:, 1::2] ** 2, y[:, 0::2] ** 2 + y[:, 1::2] ** 2, rtol=1e-6)
    back = rope.rotate(got, rope.table(-th), 32, 16)
    np.testing.assert_allclose(back, y, atol=1e-6)


def test_rope_angles_closed_form():
    from oracle import rope
    # one axis: RoFormer's theta_i = m base^(-2i/d)
    th = rope.angles(np.array([[0.0], [1.0], [7.0]]), (8,), 10000.0)
    want = np.power(10000.0, -np.arange(0, 8, 2) / 8.0)
    np.testing.assert_allclose(th, np.array([0.0, 1.0, 7.0])[:, None] * want[None, :], rtol=1e-15)
    np.testing.assert_allclose(th[1], [1.0, 0.1, 0.01, 0.001], rtol=1e-12)
    # two axes: each owns its own run of pairs and its own frequencies
    th2 = rope.angles(np.array([[2.0, 5.0]]), (4, 8), 100.0)
    np.testing.assert_allclose(th2[0], [2.0, 2.0 / 10.0, 5.0, 5.0 / np.sqrt(10.0), 5.0 / 10.0, 5.0 / 10.0 ** 1.5],
                               rtol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    # the property that makes it a position encoding: the score of a rotated
    # query and key is unchanged when both positions move by the same offset
    from oracle import rope
    g = rng(43)
    q = g.standard_normal((1, 16))
    k = g.standard_normal((1, 16))
    dims, base = (4, 6, 6), 10000.0

    def score(pq, pk):
        tq = rope.table(rope.angles(np.array([pq], np.float64), dims, base))
        tk = rope.table(rope.angles(np.array([pk], np.float64), dims, base))
        return float((rope.rotate(q, tq, 16, 16) @ rope.rotate(k, tk, 16, 16).T)[0, 0])

    s0 = score([0, 3, 9], [0, 1, 4])
    assert abs(score([5, 10, 12], [5, 8, 7]) - s0) < 1e-5
    assert abs(score([0, 4, 9], [0, 1, 4]) - s0) > 1e-3           # a different offset does change it


# ---------------------------------------------------------------- FP8 attention

@pytest.mark.parametrize("v,byte", [
    (1.0, 0x38), (-1.0, 0xB8), (448.0, 0x7E), (500.0, 0x7E), (-1e6, 0xFE), (0.0, 0x00), (-0.0, 0x80),
    (2.0 ** -9, 0x01), (-2.0 ** -9, 0x81), (2.0 ** -11, 0x00), (1.0625, 0x38), (1.1875, 0x3A), (0.875, 0x36),
    (240.0, 0x77), (3.0 * 2.0 ** -9, 0x03), (2.5 * 2.0 ** -9, 0x02),
])
def test_fp8_signed_encoding_by_hand(v, byte):
    from oracle import attention
    assert int(attention.e4m3_encode(np.array([v], np.float32))[0]) == byte


def test_fp8_encoding_against_library():
    torch = pytest.importorskip("torch")
    from oracle import attention
    g = rng(51)
    x = np.concatenate([g.standard_normal(4000) * 30.0, g.standard_normal(1000) * 0.01,
                        np.array([447.9, -447.9, 2.0 ** -10, -2.0 ** -10])]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(attention.e4m3_encode(x), want)


def test_fp8_tensor_quantiser():
    from oracle import attention
    g = rng(52)
    x = bf16_round(g.standard_normal((64, 48)).astype(np.float32) * 5.0)
    codes, s = attention.fp8_quantize(x)
    assert s == np.float32(np.float32(np.max(np.abs(x))) / np.float32(448.0))
    i = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert codes[i] & 0x7F == 0x7E                               # the largest element takes the largest code
    back = attention.fp8_dequantize(codes, s)
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -4 + float(s) * 2.0 ** -10)   # half an E4M3 step
    z, s0 = attention.fp8_quantize(np.zeros((3, 4), np.float32))
    assert s0 == 1.0 and not np.any(z)
    # a part of the tensor under the whole tensor's amax: the same scale and
    # the same bytes as those elements of the whole tensor's coding
    rest = np.delete(np.arange(64), i[0])[:6]                     # rows without the maximum
    part, sp = attention.fp8_quantize(x[rest, 10:30], amax=np.max(np.abs(x)))
    assert sp == s
    np.testing.assert_array_equal(part, codes[rest, 10:30])
    own, so = attention.fp8_quantize(x[rest, 10:30])
    assert so < s and np.any(own != part)                        # its own amax is smaller: other codes


def test_attention_two_keys_by_hand():
    from oracle import attention
    # scores (ln 3, 0): weights 3/4 and 1/4
    q = np.array([[1.0, 0.0]])
    k = np.array([[np.log(3.0), 0.0], [0.0, 0.0]])
    v = np.array([[4.0, -8.0], [8.0, 4.0]])
    o = attention.attention(q, k, v, heads=1, scale=1.0)
    np.testing.assert_allclose(o, [[0.75 * 4 + 0.25 * 8, 0.75 * -8 + 0.25 * 4]], rtol=1e-14)


def test_attention_closed_forms():
    from oracle import attention
    g = rng(53)
    S, H, d = 24, 2, 8
    q = g.standard_normal((S, H * d))
    k = g.standard_normal((S, H * d))
    v = g.standard_normal((S, H * d))
    o = attention.attention(q, k, v, H)
    # identical keys: every query averages the values
    o_u = attention.attention(q, np.ones_like(k), v, H)
    np.testing.assert_allclose(o_u, np.broadcast_to(v.mean(axis=0), o_u.shape), rtol=1e-12)
    # keys and values permuted together: unchanged; queries permuted: rows permuted
    perm = g.permutation(S)
    np.testing.assert_allclose(attention.attention(q, k[perm], v[perm], H), o, rtol=1e-12)
    np.testing.assert_allclose(attention.attention(q[perm], k, v, H), o[perm], rtol=1e-12)
    # heads are independent
    np.testing.assert_allclose(o[:, d:], attention.attention(q[:, d:], k[:, d:], v[:, d:], 1,
                                                             scale=1.0 / np.sqrt(d)), rtol=1e-12)
    # one dominant key selects its value; huge scores do not overflow
    k2 = k.copy()
    k2[5] = 1e4 * q[0]
    o2 = attention.attention(q[:1], k2, v, H)
    np.testing.assert_allclose(o2[0], v[5], atol=1e-12)
    # the scale of the scores is 1/sqrt(d) by default
    np.testing.assert_allclose(attention.attention(q, k, v, H, scale=1.0 / np.sqrt(d)), o, rtol=1e-15)
