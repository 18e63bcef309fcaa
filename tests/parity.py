"""Tolerances and error measures for comparing the CUDA path with the oracle.

The contract: relative Frobenius error <= 1e-4 for fp32 inputs; <= 5e-3 with
max-abs <= 3e-2 * RMS(reference) for bf16 inputs, on both the output and the
final state.  The reference is the unrounded fp64 oracle result.
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


def assert_close(x, ref, dtype, what=""):
    e = errors(x, ref)
    t = TOL[dtype]
    assert np.isfinite(to_f64(x)).all(), f"{what}: non-finite values"
    assert e["rel_fro"] <= t["rel_fro"], f"{what}: rel_fro {e['rel_fro']:.3e} > {t['rel_fro']:.1e}"
    if t["max_abs_rms"] is not None:
        assert e["max_abs"] <= t["max_abs_rms"] * e["rms"], (
            f"{what}: max_abs {e['max_abs']:.3e} > {t['max_abs_rms']} * rms {e['rms']:.3e}")
    return e
