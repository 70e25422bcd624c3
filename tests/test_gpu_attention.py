"""GPU parity of the FP8 attention path (fp8_quantize, attention_fp8).

* The E4M3 codes and the per-tensor scale of every quantised tensor are
  compared byte for byte with the oracle (row-major and transposed).
* Attention against the oracle's exact softmax attention of the dequantised
  tensors (fp64).  The kernel rounds the probabilities to E4M3 (3 mantissa
  bits: a relative error of up to 2^-4 per weight) before the second
  product, so on random data the output differs from the exact value by a
  few percent of its RMS; the bound below is 8e-2 in relative Frobenius norm.
  Two cases need no such allowance: identical keys (every probability is
  2^8 exactly, so O is the mean of the values) and one dominant key per
  query (every other probability underflows, so O is that key's value) --
  both checked to the bf16 rounding of the output.
* The full sequences of both block sizes (4608 tokens x 24 heads, 16896
  tokens x 48 heads): scales, the codes of sampled heads and O of sampled
  query rows against the oracle over all keys.
"""
import numpy as np
import pytest

from helpers import from_dev_bf16, to_dev_bf16
from oracle import attention as oatt
from oracle import linear as olinear
from synth import bf16_round, rng

pytestmark = pytest.mark.gpu

REL_FP8_P = 8e-2


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


@pytest.mark.parametrize("rows,cols,transpose", [(300, 384, False), (512, 256, True), (1040, 8, True)])
def test_fp8_quantize_bytes(w4, rows, cols, transpose):
    import torch
    g = rng(rows + cols)
    x = bf16_round((g.standard_normal((rows, cols)) * np.exp(g.standard_normal(cols))[None, :]).astype(np.float32))
    t = w4.quantize_fp8(to_dev_bf16(x), transpose=transpose)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    codes, s = oatt.fp8_quantize(x)
    assert float(t.scale.cpu()[0]) == float(s)
    got = t.codes.cpu().numpy()
    np.testing.assert_array_equal(got, codes.T if transpose else codes)


def run(w4, q, k, v, heads, batch):
    import torch
    tq = w4.quantize_fp8(to_dev_bf16(q))
    tk = w4.quantize_fp8(to_dev_bf16(k))
    tv = w4.quantize_fp8(to_dev_bf16(v), transpose=True)
    O = w4.attention(tq, tk, tv, heads, batch=batch)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    cq, sq = oatt.fp8_quantize(q)
    ck, sk = oatt.fp8_quantize(k)
    cv, sv = oatt.fp8_quantize(v)
    np.testing.assert_array_equal(tq.codes.cpu().numpy(), cq)
    np.testing.assert_array_equal(tk.codes.cpu().numpy(), ck)
    np.testing.assert_array_equal(tv.codes.cpu().numpy(), cv.T)
    dq, dk, dv = oatt.fp8_dequantize(cq, sq), oatt.fp8_dequantize(ck, sk), oatt.fp8_dequantize(cv, sv)
    S = q.shape[0] // batch
    ref = np.concatenate([oatt.attention(dq[b * S:(b + 1) * S], dk[b * S:(b + 1) * S], dv[b * S:(b + 1) * S], heads)
                          for b in range(batch)])
    return from_dev_bf16(O), ref


@pytest.mark.parametrize("batch,S,heads", [(1, 256, 2), (2, 384, 3), (1, 1024, 1), (3, 128, 2)])
def test_attention_random(w4, batch, S, heads):
    g = rng(100 * batch + S + heads)
    M = batch * S
    q = bf16_round(g.standard_normal((M, heads * 128)).astype(np.float32) * 1.5)
    k = bf16_round(g.standard_normal((M, heads * 128)).astype(np.float32) * 1.5)
    v = bf16_round(g.standard_normal((M, heads * 128)).astype(np.float32))
    o, ref = run(w4, q, k, v, heads, batch)
    assert np.all(np.isfinite(o))
    rel = olinear.rel_frobenius(o, ref)
    assert rel <= REL_FP8_P, f"relative Frobenius error {rel:.3e}"


def test_attention_identical_keys_give_the_mean(w4):
    g = rng(7)
    batch, S, heads = 2, 512, 2
    M = batch * S
    q = bf16_round(g.standard_normal((M, heads * 128)).astype(np.float32))
    k = np.zeros((M, heads * 128), np.float32)
    v = bf16_round(g.standard_normal((M, heads * 128)).astype(np.float32))
    o, ref = run(w4, q, k, v, heads, batch)
    assert olinear.rel_frobenius(o, ref) <= 4e-3
    assert np.max(np.abs(o - ref)) <= 2.0 ** -7 * np.max(np.abs(ref))


def test_attention_dominant_key(w4):
    """Query i < 128 and key pi(i) share one large feature (score 1024 / sqrt(128),
    130 binades above the other scores of the row, which are 0); the
    dominant keys fall in every key tile, so the running maximum moves (and O
    and l are rescaled) wherever the dominant key comes after the first tile.
    The other queries see only zero scores: O is the mean of the values."""
    g = rng(8)
    S, heads = 512, 1
    q = np.zeros((S, 128), np.float32)
    k = np.zeros((S, 128), np.float32)
    pi = g.permutation(S)
    for i in range(S):
        q[i, i % 128] = 32.0 if i < 128 else 0.0
        k[pi[i], i % 128] = 32.0 if i < 128 else 0.0    # one key per feature: the first 128 queries
    v = bf16_round(g.standard_normal((S, 128)).astype(np.float32))
    o, ref = run(w4, q, k, v, heads, 1)
    sel = np.arange(128)                                  # queries with a dominant key
    np.testing.assert_allclose(o[sel], ref[sel], rtol=2.0 ** -7, atol=2.0 ** -7 * np.max(np.abs(v)))
    rest = np.arange(128, S)                              # the others: every score 0, O = mean of V
    assert olinear.rel_frobenius(o[rest], ref[rest]) <= 4e-3


@pytest.mark.parametrize("S,heads", [(4608, 24), (16896, 48)])
def test_attention_full_size_sampled(w4, S, heads):
    """The sequences of the two block sizes (1024px: 4608 tokens, 24 heads;
    2048px: 16896 tokens, 48 heads), one sequence, in the launch the
    benchmark table times.  Every scale against the oracle's; the codes of
    sampled heads (all keys and values, sampled query rows) byte for byte
    under the whole tensor's amax; O of those rows and heads against the
    oracle's exact attention over all S keys."""
    import torch
    g = rng(9100 + S)
    D = heads * 128
    q = bf16_round(g.standard_normal((S, D), np.float32) * np.float32(1.5))
    k = bf16_round(g.standard_normal((S, D), np.float32) * np.float32(1.5))
    v = bf16_round(g.standard_normal((S, D), np.float32))
    tq = w4.quantize_fp8(to_dev_bf16(q))
    tk = w4.quantize_fp8(to_dev_bf16(k))
    tv = w4.quantize_fp8(to_dev_bf16(v), transpose=True)
    O = w4.attention(tq, tk, tv, heads)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    amax = [np.max(np.abs(a)) for a in (q, k, v)]
    for t, a in zip((tq, tk, tv), amax):
        assert float(t.scale.cpu()[0]) == float(oatt.fp8_scale(a))
    rows = np.sort(g.choice(S, 40, replace=False))
    rows[0], rows[-1] = 0, S - 1
    o_rows = from_dev_bf16(O[torch.from_numpy(rows).cuda()])
    q_rows = tq.codes[torch.from_numpy(rows).cuda()].cpu().numpy()
    for h in (0, heads // 2 + 1, heads - 1):
        cols = slice(h * 128, (h + 1) * 128)
        cq, sq = oatt.fp8_quantize(q[rows, cols], amax=amax[0])
        ck, sk = oatt.fp8_quantize(k[:, cols], amax=amax[1])
        cv, sv = oatt.fp8_quantize(v[:, cols], amax=amax[2])
        np.testing.assert_array_equal(q_rows[:, cols], cq)
        np.testing.assert_array_equal(tk.codes[:, cols].cpu().numpy(), ck)
        np.testing.assert_array_equal(tv.codes[cols].cpu().numpy(), cv.T)
        ref = oatt.attention(oatt.fp8_dequantize(cq, sq), oatt.fp8_dequantize(ck, sk),
                             oatt.fp8_dequantize(cv, sv), 1)
        o = o_rows[:, cols]
        assert np.all(np.isfinite(o))
        rel = olinear.rel_frobenius(o, ref)
        assert rel <= REL_FP8_P, f"head {h}: relative Frobenius error {rel:.3e}"
