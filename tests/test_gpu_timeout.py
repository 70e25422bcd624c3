"""A device-side wait that runs out returns an error status instead of
hanging, and the library works again once the caller has reset the status
and zeroed the workspace.

The unsatisfiable condition is set up on the host, in the caller's
workspace: the single-pass quantiser sums the low-rank partials of a row
block once its counter shows every K slice, and the counter of row block 0
starts at 2^32 - 1 instead of zero, so it stops one short of the slice
count.  With the wait bound lowered to about 25 ms, the waiting threads give
up, record W4A4_ERR_DEVICE_TIMEOUT in the sticky status word and let the
kernel end; nothing faults and no wait is unbounded.
"""
import numpy as np
import pytest

from helpers import sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4
from synth import make_linear

pytestmark = pytest.mark.gpu

TIMEOUT_STATUS = -7          # W4A4_ERR_DEVICE_TIMEOUT
TICKETS_OFFSET = 5120        # W4A4_WS_TICKETS_OFFSET
SHORT_BOUND = 50_000_000     # SM cycles, about 25 ms at 1.9 GHz


def test_wait_runs_out_and_the_library_recovers():
    import torch
    assert torch.cuda.is_available(), "GPU test"
    import bit_diffusion_transformer_nvfp4_b200 as w4
    M, K, r = 4608, 3072, 32     # 36 row blocks x 4 K slices: the single-pass path with a low-rank branch
    c = make_linear("timeout", M, K, 256, r=r, act="student_t", seed=77)
    X = to_dev_bf16(c.x)
    inv_s = to_dev_f32(np.ones(K, np.float32))
    L1t = to_dev_bf16((0.02 * np.random.default_rng(5).standard_normal((r, K))).astype(np.float32))
    t_w = to_dev_f32(np.array([0.01], np.float32))
    ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), "cuda")
    assert w4.w4a4_device_status(reset=True) == 0
    ws[TICKETS_OFFSET:TICKETS_OFFSET + 4] = 0xFF          # counter of row block 0 = 2^32 - 1
    w4.w4a4_set_wait_bound(SHORT_BOUND)
    try:
        w4.quantize_act(X, inv_s, L1t, t_w, workspace=ws)
        torch.cuda.synchronize()                          # the kernel ended on its own
        assert w4.w4a4_last_error() == TIMEOUT_STATUS     # read without a device synchronisation
        assert w4.w4a4_last_error() == TIMEOUT_STATUS     # sticky: reading does not clear it
        assert w4.w4a4_device_status(reset=True) == TIMEOUT_STATUS
        assert w4.w4a4_last_error() == 0
    finally:
        w4.w4a4_set_wait_bound(0)
    assert w4.w4a4_device_status() == 0
    # the caller zeroes the workspace after a device error; the next call is exact
    ws.zero_()
    got = w4.quantize_act(X, inv_s, L1t, t_w, workspace=ws)
    ref = w4.quantize_act(X, inv_s, L1t, t_w)             # a fresh workspace
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    oq, osf, ot, _ = nvfp4.quantize_activation(c.x, None)
    assert float(got.t_x.cpu()[0]) == float(ot)
    np.testing.assert_array_equal(got.Xq.cpu().numpy(), oq)
    np.testing.assert_array_equal(sf_atoms_to_rowmajor(got.Xsf.cpu().numpy(), M, K)[:M], osf)
    assert torch.equal(got.U, ref.U)
    u = got.U.float().cpu().numpy().astype(np.float64)
    u_ref = olinear.lowrank_down(c.x, L1t.float().cpu().numpy()) / (float(ot) * 0.01)
    assert olinear.rel_frobenius(u[:, :r] + u[:, r:], u_ref) < 1e-5
