"""The decomposition the tensor-core kernel uses for strongly decaying chunks
(the level Gram), checked in fp64 on the CPU against the direct definition of
the decayed Gram matrices (Kimi K3 digest, "Kimi Delta Attention" section:
A_rs = beta_r sum_c k_rc k_sc e^{G_rc - G_sc} for s < r, P_rs the same with
q_r, s <= r).

The scheme: level p = 64, 32, 16, 8 splits the 64 rows into aligned p-blocks;
R = G at the last row of a block's earlier half; later rows are scaled by
e^{G_r - R}, earlier rows by e^{R - G_r}; the level's Gram is kept for the
pairs whose highest differing index bit is p / 2 (finest level wins); pairs
inside one 4-row group and the diagonal are summed directly.  Without
rounding the result must equal the definition, and no factor may exceed 1
(the point of the scheme: fp16 operands never overflow at the pages' decay
bound g >= -5)."""
import numpy as np
import pytest

C, D = 64, 128


def direct(q, k, g):
    G = np.cumsum(g, axis=0)
    P = np.zeros((C, C))
    A = np.zeros((C, C))
    for r in range(C):
        for s in range(r + 1):
            e = np.exp(G[r] - G[s])
            P[r, s] = np.sum(q[r] * k[s] * e)
            if s < r:
                A[r, s] = np.sum(k[r] * k[s] * e)
    return P, A


def level_scheme(q, k, g):
    G = np.cumsum(g, axis=0)
    acc = np.zeros((2 * C, C))  # rows 0..63: P rows, 64..127: A rows (before masking)
    max_factor = 0.0
    for L in (6, 5, 4, 3):
        p = 1 << L
        X = np.zeros((2 * C, D))
        for r in range(C):
            R = G[(r & ~(p - 1)) + p // 2 - 1]
            later = (r & (p // 2)) != 0
            f = np.exp(G[r] - R) if later else np.exp(R - G[r])
            max_factor = max(max_factor, float(f.max()))
            X[r] = q[r] * f
            X[C + r] = k[r] * f
        val = X @ X[C:].T
        for ti in range(2 * C):
            r = ti % C
            for s in range(C):
                if (r >> L) == (s >> L):
                    acc[ti, s] = val[ti, s]
    for r in range(C):  # pairs inside the 4-row group of r, diagonal included
        for s in range(4 * (r // 4), r + 1):
            e = np.exp(G[r] - G[s])
            acc[r, s] = np.sum(q[r] * k[s] * e)
            acc[C + r, s] = np.sum(k[r] * k[s] * e)
    P = np.tril(acc[:C])
    A = np.tril(acc[C:], -1)
    return P, A, max_factor


def inputs(seed, gmin, valid=C):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((C, D))
    k = rng.standard_normal((C, D))
    q /= np.linalg.norm(q, axis=1, keepdims=True)
    k /= np.linalg.norm(k, axis=1, keepdims=True)
    g = gmin / (1.0 + np.exp(-rng.standard_normal((C, D))))  # g in (gmin, 0)
    q[valid:] = 0.0
    k[valid:] = 0.0
    g[valid:] = 0.0
    return q, k, g


@pytest.mark.parametrize("gmin,valid", [(-5.0 / 64.0, C), (-1.0, C), (-5.0, C), (-5.0, 37), (-5.0, 1)])
def test_level_scheme_equals_definition(gmin, valid):
    q, k, g = inputs(7, gmin, valid)
    P0, A0 = direct(q, k, g)
    P1, A1, fmax = level_scheme(q, k, g)
    assert fmax <= 1.0
    scale = max(np.abs(P0).max(), 1e-300)
    assert np.abs(P1 - P0).max() <= 1e-12 * scale
    assert np.abs(A1 - A0).max() <= 1e-12 * max(np.abs(A0).max(), 1e-300)


def test_every_pair_has_exactly_one_level():
    """Each pair s < r falls in exactly one of: a 4-row group, or the level
    p = 2^(b+1) where b is the highest bit in which r and s differ (b >= 2)."""
    for r in range(C):
        for s in range(r):
            owners = []
            if r // 4 == s // 4:
                owners.append("group")
            for L in (6, 5, 4, 3):
                p = 1 << L
                same_block = (r >> L) == (s >> L)
                straddles = (r & (p // 2)) != 0 and (s & (p // 2)) == 0
                if same_block and straddles:
                    owners.append(p)
            assert len(owners) == 1, (r, s, owners)


def test_end_reference_would_overflow_fp16_at_the_decay_bound():
    """Why the scheme exists: at g near -5 the end-of-chunk reference needs
    factors far beyond the fp16 range (65504), the level references never
    exceed 1."""
    q, k, g = inputs(3, -5.0)
    G = np.cumsum(g, axis=0)
    assert float(np.exp(G - G[-1]).max()) > 65504.0
    assert level_scheme(q, k, g)[2] <= 1.0
