"""The attention comparison's allowance for the output dtype's own rounding
(tests/gpu_helpers.half_ulp), on the CPU: it is exactly half a unit in the last
place of bf16 (8 significant bits) or fp32 (24) at the exact value's magnitude,
and a correctly rounded conversion never errs by more than it."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import gpu_helpers


def test_half_ulp_at_binade_edges():
    x = np.array([1.0, 1.999, 2.0, 7.999, 8.0, 8.43, 15.99, 0.75, 1e-3])
    want_bf16 = np.array([2.0 ** -8, 2.0 ** -8, 2.0 ** -7, 2.0 ** -6, 2.0 ** -5, 2.0 ** -5,
                          2.0 ** -5, 2.0 ** -9, 2.0 ** -18])
    assert np.array_equal(gpu_helpers.half_ulp(x, "bf16"), want_bf16)
    assert np.array_equal(gpu_helpers.half_ulp(x, "f32"), want_bf16 * 2.0 ** -16)
    assert np.array_equal(gpu_helpers.half_ulp(-x, "bf16"), want_bf16)


def test_round_to_nearest_stays_within_half_ulp():
    """fp32 -> bf16 by torch (round to nearest even): the error never exceeds the
    allowance, and reaches it at rounding midpoints."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(200_000) * np.exp2(rng.integers(-20, 12, 200_000))).astype(np.float32)
    r = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    err = np.abs(r - x.astype(np.float64))
    assert (err <= gpu_helpers.half_ulp(x.astype(np.float64), "bf16")).all()
    mid = np.float32(1.0 + 2.0 ** -8)          # halfway between two bf16 values
    rm = float(torch.tensor([mid]).to(torch.bfloat16).float())
    assert abs(rm - float(mid)) == gpu_helpers.half_ulp(np.array([1.0]), "bf16")[0]
