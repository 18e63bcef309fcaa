"""Writes tests/golden/oracle_tiny.json: a regression fixture whose inputs
are drawn with numpy's seeded generator and whose outputs come only from the
fp64 oracle (``oracle/``), itself pinned by tests/test_oracle_pins.py.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(2026)
    B, T, H, dk, dv = 1, 16, 2, 4, 3
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    g = -(5 / 64) * (1 / (1 + np.exp(-rng.standard_normal((B, T, H, dk)))))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    s0 = 0.1 * rng.standard_normal((B, H, dk, dv))
    out, fin = oracle.fwd(q, k, v, g, beta, s0)
    doc = {
        "about": "oracle regression fixture; KDA recurrence of the Kimi K3 digest, "
                 "'Kimi Delta Attention' section; inputs numpy default_rng(2026)",
        "shape": {"B": B, "T": T, "H": H, "dk": dk, "dv": dv},
        "inputs": {n: a.ravel().tolist() for n, a in
                   dict(q=q, k=k, v=v, g=g, beta=beta, init_state=s0).items()},
        "out": out.ravel().tolist(),
        "final_state": fin.ravel().tolist(),
    }
    with open(os.path.join(HERE, "oracle_tiny.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
