"""The FP4 MMA-rate measurement (w4a4_fp4_mma_rate) runs on every SM in both
modes, reports a cycle count for every issuer and leaves the status clean."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pair", [1, 0])
def test_fp4_mma_rate_runs(pair):
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_diffusion_transformer_nvfp4_b200 as w4
    w4.lib()
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    cycles = torch.zeros(n_sm, dtype=torch.int64, device="cuda")
    w4.w4a4_fp4_mma_rate(2000, pair, cycles)
    torch.cuda.synchronize()
    assert w4.w4a4_device_status() == 0
    c = cycles[: n_sm // 2 if pair else n_sm].cpu()
    assert bool((c > 0).all())
    per = c.double().median().item() / 2000
    assert 32 <= per <= 4096, per        # cycles per MMA: a plausible tensor-pipe rate
