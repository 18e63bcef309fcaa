"""The oracle reproduces its committed regression fixture bit-for-bit-ish
(fixture written by tests/golden/make_golden.py from the oracle alone)."""
import json
import os

import numpy as np

import oracle


def test_oracle_matches_golden_fixture():
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")
    doc = json.load(open(path))
    s = doc["shape"]
    B, T, H, dk, dv = s["B"], s["T"], s["H"], s["dk"], s["dv"]
    inp = {n: np.array(v) for n, v in doc["inputs"].items()}
    q = inp["q"].reshape(B, T, H, dk)
    k = inp["k"].reshape(B, T, H, dk)
    v = inp["v"].reshape(B, T, H, dv)
    g = inp["g"].reshape(B, T, H, dk)
    beta = inp["beta"].reshape(B, T, H)
    s0 = inp["init_state"].reshape(B, H, dk, dv)
    out, fin = oracle.fwd(q, k, v, g, beta, s0)
    np.testing.assert_allclose(out.ravel(), doc["out"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(fin.ravel(), doc["final_state"], rtol=1e-13, atol=1e-15)
