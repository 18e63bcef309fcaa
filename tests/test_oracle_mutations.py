"""The oracle pins must catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake (a dropped term, a flipped sign, a wrong operand, the read taken
from the pre-update state), builds it on the CPU and checks that at least
one of the pins in ``test_oracle_pins.py`` now fails.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

MUTATIONS = {
    "write_sign": ("row[j] += ki * u[j];", "row[j] -= ki * u[j];"),
    "decay_sign": ("const double a = exp(g[i]);", "const double a = exp(-g[i]);"),
    "erase_dropped": ("u[j] = beta * (v[j] - u[j]);", "u[j] = beta * v[j];"),
    "erase_sign": ("u[j] = beta * (v[j] - u[j]);", "u[j] = beta * (v[j] + u[j]);"),
    "beta_dropped": ("u[j] = beta * (v[j] - u[j]);", "u[j] = (v[j] - u[j]);"),
    "read_with_key": ("o[j] += row[j] * qi;", "o[j] += row[j] * k[i];"),
    "decay_skipped_row0": ("for (int i = 0; i < dk; ++i) {\n        const double a",
                           "for (int i = 1; i < dk; ++i) {\n        const double a"),
}

PIN_FUNCS = [
    pins.test_retrieval_orthonormal_keys_exact,
    pins.test_rewrite_same_key_replaces_value,
    pins.test_pure_channel_decay,
    pins.test_decay_acts_on_key_rows,
    pins.test_scalar_case_is_ema,
    pins.test_hand_worked_two_tokens,
    lambda: pins.test_transition_product_closed_form(8, 4, 4),
    pins.test_split_chaining_and_segment_identity,
]


def _read_before_write(src):
    """Move the read o = S^T q before the erase/write (uses S_{t-1})."""
    a = src.index("    /* read: o = S^T q")
    b = src.index("}\n\n/*\n * One (sequence, head) chain.")
    read_block = src[a:b]
    w = src.index("    /* erase + write")
    return src[:w] + read_block + src[w:a] + src[b:]


def _build_mutant(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    c.write_text(src)
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O1", "-fPIC", "-shared", "-o", str(so), str(c), "-lm",
                           "-lpthread"])
    lib = ctypes.CDLL(str(so))
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_fwd.argtypes = oracle._load().kda_oracle_fwd.argtypes
    lib.kda_oracle_decode_step.restype = None
    lib.kda_oracle_decode_step.argtypes = oracle._load().kda_oracle_decode_step.argtypes
    return lib


@pytest.mark.parametrize("name", sorted(MUTATIONS) + ["read_before_write"])
def test_pins_catch_mutation(tmp_path, name, monkeypatch):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    if name == "read_before_write":
        mutated = _read_before_write(src)
    else:
        old, new = MUTATIONS[name]
        assert old in src, f"mutation anchor for {name} not found"
        mutated = src.replace(old, new, 1)
    assert mutated != src
    lib = _build_mutant(tmp_path, name, mutated)
    monkeypatch.setattr(oracle, "_lib", lib)
    failures = 0
    for f in PIN_FUNCS:
        try:
            f()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught mutation {name}"
