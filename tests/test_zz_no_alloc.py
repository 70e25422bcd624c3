"""The allocation-free activation quantiser (nvfp4_quantize_act_noalloc).

Some hosts give a layer only its input and output buffers and no way to get
device memory: an inference-engine plugin interface without a workspace slot,
or a serving runtime that plans every buffer up front and forbids allocation
while requests run (allocating can synchronise the device and fragment the
planned pool).  For them the library carries its own scratch, a fixed-size
device array built into the shared library.

This file is named so that pytest collects it last: if it fails, a run that
stops at the first failure has already run every other test.  It passes both
on its own in a fresh process (the first call on the device then does the
one-time set-up) and after the other tests.
"""
import ctypes

import numpy as np
import pytest

from helpers import prepare, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4
from synth import bf16_round, make_linear, rng

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT_STATUS = -9  # W4A4_ERR_SCRATCH_LIMIT


def _entry(w4):
    """The C ABI function, called directly through ctypes."""
    f = w4.lib().nvfp4_quantize_act_noalloc
    P, I64 = ctypes.c_void_p, ctypes.c_int64
    f.restype = ctypes.c_int
    f.argtypes = [P, I64, I64, I64, P, P, ctypes.c_int, P, P, P, P, P, P]
    return f


def test_noalloc_matches_workspace_entry_point():
    import torch
    assert torch.cuda.is_available(), "GPU test"
    import bit_diffusion_transformer_nvfp4_b200 as w4
    f = _entry(w4)
    stream = torch.cuda.current_stream().cuda_stream
    M, K, r = 4608, 3072, 32
    # Two calls in a row with different inputs: both share the one built-in
    # scratch array, so the second call must not see stale state.
    for seed in (11, 12):
        c = make_linear("noalloc", M, K, 256, r=r, act="student_t", seed=seed)
        p = prepare(c)
        X = to_dev_bf16(c.x)
        inv_s = to_dev_f32(p["inv_s"])
        L1t = to_dev_bf16(p["L1t"])
        t_w = to_dev_f32(np.array([p["t_w"]], np.float32))
        ref = w4.quantize_act(X, inv_s, L1t, t_w)  # the entry point that takes a workspace
        Xq = torch.empty_like(ref.Xq)
        Xsf = torch.empty_like(ref.Xsf)
        t_x = torch.empty_like(ref.t_x)
        U = torch.empty_like(ref.U)
        st = f(X.data_ptr(), M, K, K, inv_s.data_ptr(), L1t.data_ptr(), r, t_w.data_ptr(),
               Xq.data_ptr(), Xsf.data_ptr(), t_x.data_ptr(), U.data_ptr(), stream)
        assert st == 0, w4.w4a4_status_string(st)
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0
        # codes, scale bytes and the tensor scale: bit for bit, against the
        # workspace entry point and against the oracle
        assert torch.equal(t_x, ref.t_x)
        assert torch.equal(Xq, ref.Xq)
        assert torch.equal(Xsf, ref.Xsf)
        oq, osf, ot, _ = nvfp4.quantize_activation(c.x, p["inv_s"])
        assert float(t_x.cpu()[0]) == float(ot)
        np.testing.assert_array_equal(Xq.cpu().numpy(), oq)
        np.testing.assert_array_equal(sf_atoms_to_rowmajor(Xsf.cpu().numpy(), M, K)[:M], osf)
        # the low-rank activations: within the tolerance the U checks use
        got = U.float().cpu().numpy().astype(np.float64)
        want = ref.U.float().cpu().numpy().astype(np.float64)
        assert olinear.rel_frobenius(got[:, :r] + got[:, r:], want[:, :r] + want[:, r:]) < 1e-5


def test_noalloc_rejects_sizes_beyond_its_scratch():
    import bit_diffusion_transformer_nvfp4_b200 as w4
    f = _entry(w4)
    fake = 1 << 20  # aligned, never dereferenced: the size check comes first
    M, K = 200_000, 3072
    assert w4.nvfp4_quant_workspace_bytes(M, K, 32) > (16 << 20)
    st = f(fake, M, K, K, None, fake, 32, fake, fake, fake, fake, fake, None)
    assert st == SCRATCH_LIMIT_STATUS
    assert "scratch" in w4.w4a4_status_string(st)


def test_noalloc_serves_calls_of_any_size_in_turn():
    """The built-in scratch is shared by every call, whatever its size: a
    sequence that crosses 64 and 128 row blocks and comes back (single-pass
    and two-pass paths) gives the workspace entry point's bytes each time,
    also after a status reset, which makes the next call zero the scratch."""
    import torch
    import bit_diffusion_transformer_nvfp4_b200 as w4
    f = _entry(w4)
    stream = torch.cuda.current_stream().cuda_stream
    K, r = 3072, 32
    t_w = to_dev_f32(np.array([0.01], np.float32))
    for i, M in enumerate([4608, 9216, 18432, 4608, "reset", 9216, 300]):
        if M == "reset":
            assert w4.w4a4_device_status(reset=True) == 0
            continue
        g = rng(1200 + i)
        x = g.standard_normal((M, K)).astype(np.float32)
        x[:, g.choice(K, 31, replace=False)] *= 60.0
        X = to_dev_bf16(bf16_round(x))
        inv_s = to_dev_f32((1.0 / np.exp(0.3 * g.standard_normal(K))).astype(np.float32))
        L1t = to_dev_bf16(bf16_round((0.02 * g.standard_normal((r, K))).astype(np.float32)))
        ref = w4.quantize_act(X, inv_s, L1t, t_w)
        Xq, Xsf = torch.empty_like(ref.Xq), torch.empty_like(ref.Xsf)
        t_x, U = torch.empty_like(ref.t_x), torch.empty_like(ref.U)
        st = f(X.data_ptr(), M, K, K, inv_s.data_ptr(), L1t.data_ptr(), r, t_w.data_ptr(),
               Xq.data_ptr(), Xsf.data_ptr(), t_x.data_ptr(), U.data_ptr(), stream)
        assert st == 0, w4.w4a4_status_string(st)
        torch.cuda.synchronize()
        assert w4.w4a4_device_status() == 0, M
        assert torch.equal(t_x, ref.t_x), M
        assert torch.equal(Xq, ref.Xq) and torch.equal(Xsf, ref.Xsf), M
        assert torch.equal(U, ref.U), M
