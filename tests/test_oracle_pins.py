"""Pins for the fp64 oracle: each check comes from the mathematics of the
gated delta rule or from a different formulation on the pages, never from
re-running the oracle's own formula.

Sources (Kimi K3 technical-report digest, discuss.pytorch.kr):
  * "Kimi Delta Attention" section: state-update equation and o_t = S_t^T q_t;
    chunkwise form (inter-chunk + intra-chunk terms).
  * "KDA algorithm-system co-design" section, KCP paragraph: the transition
    form S_t = M_t S_{t-1} + beta_t k_t v_t^T with
    M_t = (I - beta_t k_t k_t^T) Diag(alpha_t), and the segment identity
    S = S~ + M^{t<-1} S_prev (effect of a segment = zero-start state plus
    transition applied to the incoming state).
  * "Bounded decay" section: alpha_t = exp(g_t).
  * Architecture page (digitalbourgeois.tistory.com): forget / erase / write.
"""
import numpy as np
import pytest

import oracle
from chunk_model import chunk_forward

RNG = np.random.default_rng(1234)


def _rand_chain(T, dk, dv, rng, g_scale=0.5, unit=True):
    q = rng.standard_normal((T, dk))
    k = rng.standard_normal((T, dk))
    if unit:
        q /= np.linalg.norm(q, axis=1, keepdims=True)
        k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    g = -g_scale * rng.random((T, dk))
    beta = rng.random(T)
    s0 = rng.standard_normal((dk, dv)) * 0.3
    return q, k, v, g, beta, s0


def run_chain(q, k, v, g, beta, s0=None):
    """Oracle on one chain (B=1, H=1)."""
    T, dk = q.shape
    dv = v.shape[1]
    out, fin = oracle.fwd(q[None, :, None], k[None, :, None], v[None, :, None],
                          g[None, :, None], beta[None, :, None],
                          None if s0 is None else s0[None, None])
    return out[0, :, 0], fin[0, 0]


# -- 1. transition-product closed form (KCP paragraph) ----------------------
@pytest.mark.parametrize("T,dk,dv", [(1, 1, 1), (3, 2, 3), (8, 4, 4), (7, 4, 2)])
def test_transition_product_closed_form(T, dk, dv):
    rng = np.random.default_rng(T * 100 + dk * 10 + dv)
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dv, rng, unit=False)
    M = [(np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) for t in range(T)]

    def prod(a, b):  # M_b ... M_{a}  (later transitions on the left)
        P = np.eye(dk)
        for s in range(a, b + 1):
            P = M[s] @ P
        return P

    for t in range(T):
        # S_t = (M_t..M_0) S_0 + sum_{u<=t} (M_t..M_{u+1}) beta_u k_u v_u^T
        S_t = prod(0, t) @ s0 + sum(prod(u + 1, t) @ (beta[u] * np.outer(k[u], v[u]))
                                    for u in range(t + 1))
        out, fin = run_chain(q[:t + 1], k[:t + 1], v[:t + 1], g[:t + 1], beta[:t + 1], s0)
        np.testing.assert_allclose(fin, S_t, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(out[t], S_t.T @ q[t], rtol=1e-12, atol=1e-12)


# -- 2. delta-rule retrieval: erase-then-write semantics --------------------
def test_retrieval_orthonormal_keys_exact():
    d = 8
    rng = np.random.default_rng(7)
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    keys = Qm.T                        # orthonormal rows
    vals = rng.standard_normal((d, d))
    g = np.zeros((d, d))               # alpha = 1
    beta = np.ones(d)                  # full write strength
    out, fin = run_chain(keys.copy(), keys, vals, g, beta, None)
    # querying with the key just written returns its value (o uses S_t)
    np.testing.assert_allclose(out, vals, atol=1e-12)
    # after all writes every key still retrieves its own value
    np.testing.assert_allclose(keys @ fin, vals, atol=1e-12)


def test_rewrite_same_key_replaces_value():
    d = 4
    k1 = np.array([1.0, 0, 0, 0])
    k2 = np.array([0, 1.0, 0, 0])
    v1, v1b, v2 = np.array([1.0, 2, 3, 4]), np.array([-5.0, 6, 0, 1]), np.array([9.0, 9, 9, 9])
    K = np.stack([k1, k2, k1])
    V = np.stack([v1, v2, v1b])
    out, fin = run_chain(K.copy(), K, V, np.zeros((3, d)), np.ones(3), None)
    np.testing.assert_allclose(fin.T @ k1, v1b, atol=1e-12)   # replaced, not summed
    np.testing.assert_allclose(fin.T @ k2, v2, atol=1e-12)    # untouched


# -- 3. pure decay (beta = 0) -------------------------------------------------
def test_pure_channel_decay():
    T, dk, dv = 9, 5, 3
    rng = np.random.default_rng(3)
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dv, rng, g_scale=2.0)
    beta[:] = 0.0
    out, fin = run_chain(q, k, v, g, beta, s0)
    np.testing.assert_allclose(fin, np.exp(g.sum(0))[:, None] * s0, rtol=1e-12, atol=1e-14)
    for t in range(T):
        St = np.exp(g[:t + 1].sum(0))[:, None] * s0
        np.testing.assert_allclose(out[t], St.T @ q[t], rtol=1e-12, atol=1e-14)


def test_decay_acts_on_key_rows():
    # dk=2, dv=3, S0 = ones; halve channel 0, quarter channel 1; no write.
    s0 = np.ones((2, 3))
    g = np.log(np.array([[0.5, 0.25]]))
    out, fin = run_chain(np.array([[1.0, 0.0]]), np.zeros((1, 2)), np.zeros((1, 3)), g,
                         np.zeros(1), s0)
    np.testing.assert_allclose(fin, [[0.5] * 3, [0.25] * 3], atol=1e-15)
    np.testing.assert_allclose(out[0], [0.5] * 3, atol=1e-15)


# -- 4. scalar state: exponential moving average ----------------------------
def test_scalar_case_is_ema():
    T = 20
    rng = np.random.default_rng(11)
    kk = np.where(rng.random(T) < 0.5, -1.0, 1.0)
    v = rng.standard_normal(T)
    q = rng.standard_normal(T)
    g = -rng.random(T)
    beta = rng.random(T)
    s = 0.7
    expect_o = []
    for t in range(T):  # k^2 = 1: s <- (1 - beta) alpha s + beta k v
        s = (1 - beta[t]) * np.exp(g[t]) * s + beta[t] * kk[t] * v[t]
        expect_o.append(s * q[t])
    out, fin = run_chain(q[:, None], kk[:, None], v[:, None], g[:, None], beta, np.array([[0.7]]))
    np.testing.assert_allclose(out[:, 0], expect_o, rtol=1e-12)
    np.testing.assert_allclose(fin[0, 0], s, rtol=1e-12)


# -- 5. a hand-worked two-token example --------------------------------------
def test_hand_worked_two_tokens():
    # t=1: k=(1,0), v=(2,3), beta=.5, alpha=(1,1): S1 = .5 k v^T = [[1,1.5],[0,0]]
    #      q=(1,1): o1 = (1, 1.5)
    # t=2: alpha=(.5,1): S' = [[.5,.75],[0,0]]; k=(.6,.8): u = S'^T k = (.3,.45)
    #      v=(1,-1), beta=.5: delta = .5 (v-u) = (.35,-.725)
    #      S2 = S' + k delta^T = [[.71,.315],[.28,-.58]]; q=(0,1): o2 = (.28,-.58)
    q = np.array([[1.0, 1.0], [0.0, 1.0]])
    k = np.array([[1.0, 0.0], [0.6, 0.8]])
    v = np.array([[2.0, 3.0], [1.0, -1.0]])
    g = np.log(np.array([[1.0, 1.0], [0.5, 1.0]]))
    beta = np.array([0.5, 0.5])
    out, fin = run_chain(q, k, v, g, beta, None)
    np.testing.assert_allclose(out, [[1.0, 1.5], [0.28, -0.58]], atol=1e-14)
    np.testing.assert_allclose(fin, [[0.71, 0.315], [0.28, -0.58]], atol=1e-14)


# -- 6. chaining / segment identity ----------------------------------------
def test_split_chaining_and_segment_identity():
    T, dk, dv = 50, 6, 5
    rng = np.random.default_rng(5)
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dv, rng)
    out, fin = run_chain(q, k, v, g, beta, s0)
    T1 = 23
    o1, mid = run_chain(q[:T1], k[:T1], v[:T1], g[:T1], beta[:T1], s0)
    o2, fin2 = run_chain(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], mid)
    np.testing.assert_allclose(np.concatenate([o1, o2]), out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(fin2, fin, rtol=1e-12, atol=1e-13)
    # segment identity: S = S~ + M S_prev, with S~ from a zero start and M
    # the segment's transition (read off by starting from the identity
    # columns with v = 0).
    _, S_tilde = run_chain(q[T1:], k[T1:], v[T1:], g[T1:], beta[T1:], np.zeros((dk, dv)))
    _, Mseg = run_chain(q[T1:], k[T1:], np.zeros((T - T1, dk)), g[T1:], beta[T1:], np.eye(dk))
    np.testing.assert_allclose(S_tilde + Mseg @ mid, fin, rtol=1e-11, atol=1e-12)


def test_packed_equals_separate():
    rng = np.random.default_rng(9)
    H, dk, dv = 3, 4, 5
    lens = [7, 0, 13, 1, 20]
    Tt = sum(lens)
    q, k, v, g, beta = (rng.standard_normal((1, Tt, H, d)) for d in (dk, dk, dv, dk, 1))
    g = -np.abs(g)
    beta = 1 / (1 + np.exp(-beta[..., 0]))
    init = rng.standard_normal((len(lens), H, dk, dv))
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, fin = oracle.fwd(q, k, v, g, beta, init, cu_seqlens=cu)
    for n, L in enumerate(lens):
        s = slice(cu[n], cu[n + 1])
        o_n, f_n = oracle.fwd(q[:, s], k[:, s], v[:, s], g[:, s], beta[:, s], init[n:n + 1])
        np.testing.assert_allclose(out[:, s], o_n, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(fin[n], f_n[0], rtol=1e-13, atol=1e-13)
    np.testing.assert_array_equal(fin[1], init[1])   # empty sequence: final = init


# -- 7. linearity in (v, S0) --------------------------------------------------
def test_linearity_in_values_and_state():
    T, dk, dv = 30, 5, 4
    rng = np.random.default_rng(21)
    q, k, v1, g, beta, s1 = _rand_chain(T, dk, dv, rng)
    v2 = rng.standard_normal((T, dv))
    s2 = rng.standard_normal((dk, dv))
    oa, fa = run_chain(q, k, v1, g, beta, s1)
    ob, fb = run_chain(q, k, v2, g, beta, s2)
    oc, fc = run_chain(q, k, v1 + 2.5 * v2, g, beta, s1 + 2.5 * s2)
    np.testing.assert_allclose(oc, oa + 2.5 * ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(fc, fa + 2.5 * fb, rtol=1e-11, atol=1e-12)


# -- 8. contraction bound ------------------------------------------------------
def test_contraction_bound():
    T, dk, dv = 40, 8, 6
    rng = np.random.default_rng(4)
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dv, rng)
    S = s0
    for t in range(T):
        _, S_new = run_chain(q[t:t + 1], k[t:t + 1], v[t:t + 1], g[t:t + 1], beta[t:t + 1], S)
        assert np.linalg.norm(S_new) <= np.linalg.norm(S) + beta[t] * np.linalg.norm(v[t]) + 1e-12
        S = S_new


# -- 9. decode step == one-token forward --------------------------------------
def test_decode_steps_equal_forward():
    B, H, dk, dv, T = 2, 3, 4, 5, 6
    rng = np.random.default_rng(17)
    q, k, v, g = (rng.standard_normal((B, T, H, d)) for d in (dk, dk, dv, dk))
    g = -np.abs(g) * 0.3
    beta = rng.random((B, T, H))
    s0 = rng.standard_normal((B, H, dk, dv))
    out, fin = oracle.fwd(q, k, v, g, beta, s0)
    state = s0.copy()
    for t in range(T):
        o_t = oracle.decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], state)
        np.testing.assert_allclose(o_t, out[:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(state, fin, rtol=1e-12, atol=1e-13)


# -- 10. the chunk-form model (test aid) agrees with the oracle --------------
@pytest.mark.parametrize("T,C,g_scale", [(64, 16, 0.1), (150, 64, 0.08), (100, 32, 5.0)])
def test_chunk_form_matches_oracle(T, C, g_scale):
    rng = np.random.default_rng(T + C)
    q, k, v, g, beta, s0 = _rand_chain(T, 16, 12, rng, g_scale=g_scale)
    out, fin = run_chain(q, k, v, g, beta, s0)
    O, S = chunk_forward(q, k, v, g, beta, s0, C=C)
    np.testing.assert_allclose(O, out, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S, fin, rtol=1e-10, atol=1e-10)


# -- segment transition and transformed queries (KCP paragraph) -------------
@pytest.mark.parametrize("T,dk", [(1, 2), (5, 3), (8, 4)])
def test_transition_is_the_product_of_token_transitions(T, dk):
    """oracle.transition against explicit products of M_t = (I - b k k^T) Diag(e^g):
    M = M_T ... M_1 and qhat_t = (M_t ... M_1)^T q_t."""
    rng = np.random.default_rng(10 * T + dk)
    q, k, _, g, beta, _ = _rand_chain(T, dk, dk, rng, unit=False)
    qhat, M = oracle.transition(q[None, :, None], k[None, :, None], g[None, :, None], beta[None, :, None])
    P = np.eye(dk)
    for t in range(T):
        P = (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(g[t])) @ P
        np.testing.assert_allclose(qhat[0, t, 0], P.T @ q[t], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(M[0, 0], P, rtol=1e-12, atol=1e-12)


def test_segment_outputs_are_zero_start_plus_transformed_query_read():
    """Within a segment entered with state S_in: o_t = o~_t + S_in^T qhat_t and
    S_end = S~ + M S_in (linearity of the recurrence in the incoming state)."""
    rng = np.random.default_rng(99)
    T, dk = 37, 6
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dk, rng)
    o_full, s_full = run_chain(q, k, v, g, beta, s0)
    o_zero, s_zero = run_chain(q, k, v, g, beta, None)
    qhat, M = oracle.transition(q[None, :, None], k[None, :, None], g[None, :, None], beta[None, :, None])
    np.testing.assert_allclose(o_zero + qhat[0, :, 0] @ s0, o_full, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s_zero + M[0, 0] @ s0, s_full, rtol=1e-11, atol=1e-12)


def test_composition_over_many_segments():
    """A sequence cut into 4 pieces: the prefix composition of the pieces'
    (M, S~) reproduces the states at every cut and the final state."""
    rng = np.random.default_rng(5)
    T, dk = 60, 4
    q, k, v, g, beta, s0 = _rand_chain(T, dk, dk, rng)
    cuts = [0, 7, 20, 41, 60]
    S = s0
    for a, b in zip(cuts[:-1], cuts[1:]):
        _, s_zero = run_chain(q[a:b], k[a:b], v[a:b], g[a:b], beta[a:b], None)
        _, M = oracle.transition(q[None, a:b, None], k[None, a:b, None], g[None, a:b, None], beta[None, a:b, None])
        S = s_zero + M[0, 0] @ S
        _, s_ref = run_chain(q[:b], k[:b], v[:b], g[:b], beta[:b], s0)
        np.testing.assert_allclose(S, s_ref, rtol=1e-10, atol=1e-12)


# -- the input prologue (KDA section: L2 norm of q, k; Bounded decay: the gate) --
def test_gate_closed_forms():
    """g = g_min sigmoid(e^A z): g(0) = g_min / 2; g -> g_min for z -> +inf and
    -> 0 for z -> -inf; e^A scales z; always inside (g_min, 0)."""
    H, d = 3, 5
    A = np.array([0.0, np.log(2.0), -1.0])
    z0 = np.zeros((4, H, d))
    np.testing.assert_allclose(oracle.gate(z0, A), -2.5, rtol=0, atol=0)
    assert np.all(oracle.gate(z0 + 200.0, A) < -5.0 + 1e-12)
    assert np.all(oracle.gate(z0 - 200.0, A) > -1e-12)
    rng = np.random.default_rng(3)
    z = rng.standard_normal((4, H, d))
    g = oracle.gate(z, A)
    assert np.all((g > -5.0) & (g < 0.0))
    np.testing.assert_allclose(g[:, 1], oracle.gate(2.0 * z, np.zeros(H))[:, 1], rtol=1e-15)
    np.testing.assert_allclose(oracle.gate(z, A, g_min=-3.0), g * 0.6, rtol=1e-15)
    # monotone decreasing in z (a larger logit decays more)
    zs = np.sort(rng.standard_normal(50))
    gs = oracle.gate(zs[:, None, None] * np.ones((1, H, d)), A)[:, 0, 0]
    assert np.all(np.diff(gs) < 0)


def test_l2norm_unit_rows_and_direction():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 3, 16)) * rng.uniform(0.1, 10.0, (7, 3, 1))
    y = oracle.l2norm(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=0, atol=1e-6)
    cos = (x * y).sum(-1) / np.linalg.norm(x, axis=-1) / np.linalg.norm(y, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=0, atol=1e-14)


def test_gated_forward_ignores_the_scale_of_q_and_k():
    """Normalising q and k makes the output blind to their per-token scale."""
    rng = np.random.default_rng(8)
    B, T, H, d = 1, 20, 2, 8
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    v = rng.standard_normal((B, T, H, d))
    z = rng.standard_normal((B, T, H, d))
    beta = rng.random((B, T, H))
    A = np.array([0.3, -0.2])
    o1, s1 = oracle.fwd_gated(q, k, v, z, A, beta)
    o2, s2 = oracle.fwd_gated(q * rng.uniform(0.5, 3.0, (B, T, H, 1)), k * rng.uniform(0.5, 3.0, (B, T, H, 1)),
                              v, z, A, beta)
    np.testing.assert_allclose(o2, o1, rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(s2, s1, rtol=1e-5, atol=1e-7)


# -- speculative verification with state replay (serving section) -----------
def test_spec_decode_equals_forward_over_the_accepted_tokens():
    """Outputs of the new window = outputs of a forward over the accepted
    drafts followed by the new window; the kept state = that forward's state
    after the bonus token; rejected drafts leave no trace."""
    rng = np.random.default_rng(12)
    B, Wp, W, H, d = 4, 3, 4, 2, 6
    mk = lambda n: dict(q=rng.standard_normal((B, n, H, d)), k=rng.standard_normal((B, n, H, d)),
                        v=rng.standard_normal((B, n, H, d)), g=-0.3 * rng.random((B, n, H, d)),
                        beta=rng.random((B, n, H)))
    prev, cur = mk(Wp), mk(W)
    s0 = 0.2 * rng.standard_normal((B, H, d, d))
    na = np.array([0, 1, 3, 2])
    st = s0.copy()
    out = oracle.spec_decode(prev, na, cur, st)
    for b in range(B):
        cat = {n: np.concatenate([prev[n][b:b + 1, :na[b]], cur[n][b:b + 1]], 1) for n in prev}
        o_ref, _ = oracle.fwd(cat["q"], cat["k"], cat["v"], cat["g"], cat["beta"], s0[b:b + 1])
        np.testing.assert_allclose(out[b], o_ref[0, na[b]:], rtol=1e-12, atol=1e-12)
        upto = {n: v[:, :na[b] + 1] for n, v in cat.items()}
        _, s_ref = oracle.fwd(upto["q"], upto["k"], upto["v"], upto["g"], upto["beta"], s0[b:b + 1])
        np.testing.assert_allclose(st[b], s_ref[0], rtol=1e-12, atol=1e-12)
