"""One workspace, zeroed once, serves any sequence of calls.

The quantiser's per-row-block tickets of the low-rank sums (zero at rest:
every call clears what it used) and the single-pass grid barrier (a launch
generation that every call advances, with a counter and a maximum word per
generation parity) live at fixed offsets of the caller's workspace, whatever
the call's sizes.  Here one shared workspace runs the single-pass
cooperative path, the two-pass path (an activation too large to be
co-resident) and the quantise-with-given-amax path, in an order that changes
the grid size and the number of row blocks between calls, across 64 and 128
row blocks and back (a layout that moved with M would put one call's
low-rank partial sums on another call's counters); every result must equal
the oracle's bytes (small shapes) or a fresh-workspace call's bytes (large
shapes), and the device status must stay clean.
"""
import numpy as np
import pytest

from helpers import sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import nvfp4
from synth import bf16_round, rng

pytestmark = pytest.mark.gpu

SEQ = [  # (M, K, r, path)
    (4608, 3072, 32, "measured"),    # single pass, 144 CTAs
    (300, 512, 32, "measured"),      # single pass, 3 row blocks
    (4608, 12288, 32, "measured"),   # two passes (tile set not co-resident)
    (257, 768, 0, "measured"),       # single pass, no low-rank branch
    (300, 512, 32, "given"),         # quantise pass only, tickets used
    (4608, 3072, 32, "measured"),    # single pass again after all of the above
    (4608, 3072, 32, "given"),
    (128, 3072, 32, "measured"),
    (9216, 3072, 32, "measured"),    # 72 row blocks: two passes
    (18432, 3072, 32, "measured"),   # 144 row blocks
    (4608, 3072, 32, "measured"),    # 36 row blocks again: single pass
    (18432, 3072, 32, "given"),
    (9216, 3072, 16, "measured"),
    (300, 512, 32, "measured"),
]


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


def _inputs(i, M, K, r):
    g = rng(700 + i)
    x = g.standard_normal((M, K)).astype(np.float32)
    x[:, g.choice(K, max(1, K // 100), replace=False)] *= 50.0
    x = bf16_round(x)
    inv_s = (1.0 / np.exp(0.3 * g.standard_normal(K))).astype(np.float32)
    L1t = bf16_round((g.standard_normal((32, K)) * 0.02).astype(np.float32)) if r else None
    return x, inv_s, L1t


def test_one_workspace_many_calls(w4):
    import torch
    ws = w4.new_workspace(max(w4.nvfp4_quant_workspace_bytes(M, K, r) for M, K, r, _ in SEQ), "cuda")
    t_w = to_dev_f32(np.array([0.01], np.float32))
    for i, (M, K, r, path) in enumerate(SEQ):
        x, inv_s, L1t = _inputs(i, M, K, r)
        X, S = to_dev_bf16(x), to_dev_f32(inv_s)
        L = to_dev_bf16(L1t) if r else None
        T = t_w if r else None
        amax = None
        if path == "given":
            a = np.max(np.abs((x * inv_s[None, :]).astype(np.float32)))
            amax = to_dev_f32(np.array([a], np.float32))
        got = w4.quantize_act(X, S, L, T, amax=amax, workspace=ws)
        ref = w4.quantize_act(X, S, L, T, amax=amax)  # a fresh workspace
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0, (i, M, K, r, path)
        assert torch.equal(got.Xq, ref.Xq) and torch.equal(got.Xsf, ref.Xsf), (i, M, K, r, path)
        assert torch.equal(got.t_x, ref.t_x), (i, M, K, r, path)
        if r:
            assert torch.equal(got.U, ref.U), (i, M, K, r, path)
        if M * K <= 300 * 768:
            oq, osf, ot, _ = nvfp4.quantize_activation(x, inv_s)
            assert float(got.t_x.cpu()[0]) == float(ot)
            np.testing.assert_array_equal(got.Xq.cpu().numpy(), oq)
            np.testing.assert_array_equal(sf_atoms_to_rowmajor(got.Xsf.cpu().numpy(), M, K)[:M], osf)
