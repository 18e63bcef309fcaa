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


def test_error_accumulator_matches_one_shot_measures():
    import pytest
    from parity import ErrorAccumulator, assert_close, errors
    rng = np.random.default_rng(1)
    ref = rng.standard_normal((4, 50, 6))
    x = ref + 1e-3 * rng.standard_normal(ref.shape)
    acc = ErrorAccumulator(torch.bfloat16, "pieces")
    for h in range(6):
        acc.add(x[:, :, h], ref[:, :, h])
    e = acc.check()
    e1 = errors(x, ref)
    assert abs(e["rel_fro"] - e1["rel_fro"]) < 1e-12 * e1["rel_fro"] + 1e-15
    assert e["max_abs"] == e1["max_abs"] and abs(e["rms"] - e1["rms"]) < 1e-12
    # the literal max-abs bound fails where one element is off by more than 3e-2 RMS
    y = x.copy()
    y[0, 0, 0] += 0.05
    bad = ErrorAccumulator(torch.bfloat16, "pieces")
    bad.add(y, ref)
    with pytest.raises(AssertionError):
        bad.check()
    with pytest.raises(AssertionError):
        assert_close(y, ref, torch.bfloat16, literal=True)


def test_auto_reading_follows_the_rounding_of_the_exact_result():
    from parity import assert_close, rounding_alone
    rng = np.random.default_rng(2)
    calm = rng.standard_normal(4000)                       # max ~ 3.7 RMS: rounding alone ~0.007 RMS
    assert rounding_alone(calm) < 0.02
    e = assert_close(torch.from_numpy(calm).to(torch.bfloat16), calm, torch.bfloat16, literal="auto")
    assert e["literal"]
    heavy = np.concatenate([rng.standard_normal(4000) * 0.05, [7.9, -7.9]])  # max ~ 50 RMS
    assert rounding_alone(heavy) > 0.03
    e = assert_close(torch.from_numpy(heavy).to(torch.bfloat16), heavy, torch.bfloat16, literal="auto")
    assert not e["literal"]
