"""GPU parity on the 2048px workload shapes (the largest configuration):
fused QKV + MLP-up 6144 -> 55296 and the output projection 24576 -> 6144, at
2112 tokens (a ragged 17th row block) with full K and N.

The GPU packs the whole residual itself; the sampled weight rows are checked
bit for bit against the oracle's quantiser (under the whole residual's tensor
scale), then Y on sampled tokens x sampled output channels against the
oracle's fp64 result from those same oracle bytes.  The 24576-deep projection
needs more K slices than can be co-resident, so it also runs the two-pass
activation quantiser on bf16 input.
"""
import numpy as np
import pytest

from helpers import check_y, from_dev_bf16, sf_atoms_to_rowmajor, to_dev_bf16, to_dev_f32
from oracle import linear as olinear
from oracle import nvfp4, prep
from synth import config_cases, rng

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def w4():
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w
    w.lib()
    return w


@pytest.fixture(scope="module")
def cases():
    return config_cases(4, scale_m=0.125)


@pytest.mark.parametrize("which", [0, 1])
def test_config4_sampled(w4, cases, which):
    import torch
    c = cases[which]
    p = prep.svdquant_prepare(c.w, c.x_cal, c.r, c.alpha)
    g = rng(4000 + which)
    rows = np.sort(g.choice(c.M, 96, replace=False))
    rows[-1] = c.M - 1                           # the ragged last row block
    cols = np.sort(g.choice(c.N, 384, replace=False))
    cols[-1] = c.N - 1

    # the GPU packs the whole residual
    pw = w4.pack_weight(to_dev_f32(p["R"]))
    torch.cuda.synchronize()
    # oracle bytes of the sampled weight rows under the whole residual's scale
    oq, osf, ot, _ = nvfp4.quantize(p["R"][cols], amax=np.max(np.abs(p["R"])))
    owq = nvfp4.pack(oq)
    assert float(pw.t_w.cpu()[0]) == float(ot)
    gwq = pw.Wq.cpu().numpy()[cols]
    gsf = sf_atoms_to_rowmajor(pw.Wsf.cpu().numpy(), c.N, c.K)[cols]
    np.testing.assert_array_equal(gwq, owq)
    np.testing.assert_array_equal(gsf, osf)

    w = w4.PackedWeight(pw.Wq, pw.Wsf, pw.t_w, c.N, c.K, to_dev_f32(p["inv_s"]), to_dev_bf16(p["L1t"]),
                        to_dev_bf16(p["L2t"]), to_dev_bf16(c.bias) if c.bias is not None else None)
    Y = w4.linear(to_dev_bf16(c.x), w)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    y = from_dev_bf16(Y)[rows][:, cols]
    y_ref, _ = olinear.w4a4_linear(c.x, p["inv_s"], owq, osf, ot, p["L1t"], p["L2t"][cols],
                                   None if c.bias is None else c.bias[cols], rows=rows)
    check_y(y, y_ref)
