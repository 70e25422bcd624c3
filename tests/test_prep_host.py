"""Host-side checks of the weight and table preparation helpers (no GPU):
the SwiGLU row order and the rotary-embedding table against the oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import rope as orope
from synth import token_positions


def test_rope_table_matches_the_oracle_on_the_host():
    from bit_diffusion_transformer_nvfp4_b200 import prep
    pos = token_positions(64, 16, 16)
    for axes in ((16, 56, 56), (8, 12, 12)):
        got = prep.rope_table(torch.from_numpy(pos), axes).numpy()
        want = orope.table(orope.angles(pos, axes, 10000.0))
        assert got.dtype == np.float32 and got.shape == want.shape
        np.testing.assert_array_equal(got, want)
    # one axis, another base
    p1 = np.arange(50)
    np.testing.assert_array_equal(prep.rope_table(torch.from_numpy(p1), (32,), base=500.0).numpy(),
                                  orope.table(orope.angles(p1, (32,), 500.0)))
    with pytest.raises(ValueError):
        prep.rope_table(torch.from_numpy(pos), (16, 56))          # one feature count per axis
    with pytest.raises(ValueError):
        prep.rope_table(torch.from_numpy(pos), (15, 57, 56))      # even counts only


def test_swiglu_row_order_is_a_permutation_pairing_gate_and_up():
    from bit_diffusion_transformer_nvfp4_b200 import prep
    n_plain, n_ff = 64, 48
    order = prep.swiglu_row_order(n_plain, n_ff).numpy()
    assert sorted(order.tolist()) == list(range(n_plain + 2 * n_ff))
    np.testing.assert_array_equal(order[:n_plain], np.arange(n_plain))
    tail = order[n_plain:].reshape(-1, 32)
    for b, blk in enumerate(tail):           # per 16 features: their 16 gate rows, then their 16 up rows
        np.testing.assert_array_equal(blk[:16], n_plain + 16 * b + np.arange(16))
        np.testing.assert_array_equal(blk[16:], n_plain + n_ff + 16 * b + np.arange(16))
    with pytest.raises(ValueError):
        prep.swiglu_row_order(0, 40)
