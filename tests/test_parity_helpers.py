"""The tolerance helper's half-ulp allowance is exactly the bf16 rounding bound."""
import numpy as np
import torch

from parity import half_ulp_bf16


def test_half_ulp_bounds_bf16_rounding():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        [1.0, 2.0, 0.75, -3.5, 1e-30]])
    xb = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    err = np.abs(xb - x)
    hu = half_ulp_bf16(x)
    assert (err <= hu * (1 + 1e-12)).all()
    # and the bound is tight: some values sit close to a midpoint
    assert (err > 0.9 * hu).any()
    assert half_ulp_bf16(np.array([1.0]))[0] == 2.0 ** -8
    assert half_ulp_bf16(np.array([0.0]))[0] == 0.0
