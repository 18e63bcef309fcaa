"""fp64 chunk-form model of the KDA forward pass (a test aid, not the oracle).

It evaluates the chunkwise-parallel form from the Kimi K3 digest, section
"Kimi Delta Attention" (chunk output = inter-chunk term (Gamma ⊙ Q) S plus an
intra-chunk term A Ṽ), written out per chunk of C tokens with the WY/UT
factors the CUDA kernels compute:

  G_r = sum_{s<=r} g_s            (per key channel, within the chunk)
  A_rs = beta_r sum_c k_rc k_sc exp(G_rc - G_sc)    for s < r
  P_rs = sum_c q_rc k_sc exp(G_rc - G_sc)           for s <= r
  T = (I + A)^-1,  U = T diag(beta) V,  W = T diag(beta) (K ⊙ exp(G))
  Delta = U - W S
  O = (Q ⊙ exp(G)) S + P Delta
  S <- Diag(exp(G_C)) S + (K ⊙ exp(G_C - G))^T Delta

The pairwise decays are formed directly as exp(G_rc - G_sc) (no
factorisation), so this model has no overflow concerns.  It is checked
against the oracle in ``test_oracle_pins.py`` and gives the intermediates
that GPU debugging compares against.
"""
import numpy as np


def chunk_forward(q, k, v, g, beta, s0=None, C=64, keep=False):
    """One (sequence, head) chain.  q,k,g [T,dk]; v [T,dv]; beta [T]."""
    q, k, v, g, beta = (np.asarray(x, np.float64) for x in (q, k, v, g, beta))
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if s0 is None else np.array(s0, np.float64)
    O = np.zeros((T, dv))
    inter = []
    for c0 in range(0, T, C):
        sl = slice(c0, min(T, c0 + C))
        Q, K, V, Gl, b = q[sl], k[sl], v[sl], g[sl], beta[sl]
        n = Q.shape[0]
        G = np.cumsum(Gl, axis=0)
        D = G[:, None, :] - G[None, :, :]          # D[r,s,c] = G_rc - G_sc
        lower = np.tril(np.ones((n, n)), -1)
        lower_eq = np.tril(np.ones((n, n)))
        E = np.exp(np.where(lower_eq[:, :, None] > 0, D, 0.0))
        A = b[:, None] * np.einsum("rc,sc,rsc->rs", K, K, E) * lower
        P = np.einsum("rc,sc,rsc->rs", Q, K, E) * lower_eq
        Tm = np.linalg.inv(np.eye(n) + A)
        U = Tm @ (b[:, None] * V)
        W = Tm @ (b[:, None] * (K * np.exp(G)))
        Delta = U - W @ S
        O[sl] = (Q * np.exp(G)) @ S + P @ Delta
        if keep:
            inter.append(dict(G=G, A=A, P=P, T=Tm, U=U, W=W, Delta=Delta, S_in=S.copy()))
        S = np.exp(G[-1])[:, None] * S + (K * np.exp(G[-1][None, :] - G)).T @ Delta
    return (O, S, inter) if keep else (O, S)
