"""KCP host logic as world_size-2 gloo ranks on CPU: each rank holds one
consecutive slice of every sequence, the pieces (M, S~) travel through one
fixed-size all-gather, and the composed incoming state gives each rank's
outputs and the sequence's final state.  The pieces are computed here by the
fp64 oracle and the composition / correction by their definitions, so what
is tested is the rank bookkeeping of gated_delta_rule_121_b200.kcp (which
rank holds which piece, the order of the gathered pieces, the init state on
the first rank); the CUDA kernels behind the same steps are tested on the GPU
(tests/test_gpu_segments.py)."""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B=2, T=50, H=2, d=4, seed=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, d))
    k = rng.standard_normal((B, T, H, d))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, d))
    g = -0.3 * rng.random((B, T, H, d))
    beta = rng.random((B, T, H))
    init = 0.2 * rng.standard_normal((B, H, d, d))
    return q, k, v, g, beta, init


def _oracle_ops():
    import oracle

    def segment_fwd(q, k, v, g, beta):
        o, s = oracle.fwd(q, k, v, g, beta, None)
        qh, M = oracle.transition(q, k, g, beta)
        t = lambda a: torch.from_numpy(a)
        return t(o), t(s), t(qh), t(M)

    def state_compose(trans, s0, R, init_state=None, rank_major=False):
        P, H, dk, dv = s0.shape
        N = P // R
        idx = (lambda m, r: r * N + m) if rank_major else (lambda m, r: m * R + r)
        state_in = torch.zeros_like(s0)
        fin = torch.zeros((N, H, dk, dv), dtype=s0.dtype)
        for m in range(N):
            cur = init_state[m].clone() if init_state is not None else torch.zeros((H, dk, dv), dtype=s0.dtype)
            for r in range(R):
                p = idx(m, r)
                state_in[p] = cur
                cur = s0[p] + trans[p] @ cur
            fin[m] = cur
        return state_in, fin

    def output_correct(out_zero, qhat, state_in, dtype=None):
        return out_zero + torch.einsum("bthi,bhij->bthj", qhat, state_in)

    return types.SimpleNamespace(segment_fwd=segment_fwd, state_compose=state_compose,
                                 output_correct=output_correct)


def _rank_main(rank, world, port, cuts, q_out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    from gated_delta_rule_121_b200 import kcp
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        q, k, v, g, beta, init = (torch.from_numpy(a) for a in _inputs())
        a, b = cuts[rank], cuts[rank + 1]
        sl = lambda t: t[:, a:b].contiguous()
        out, fin = kcp.kcp_fwd(sl(q), sl(k), sl(v), sl(g), sl(beta), init, ops=_oracle_ops())
        q_out.put((rank, out.numpy(), fin.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 23, 50], [0, 1, 50], [0, 50, 50]])
def test_kcp_two_ranks_matches_single_sequence_oracle(cuts):
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, cuts, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, out, fin = q_out.get(timeout=120)
        res[r] = (out, fin)
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    q, k, v, g, beta, init = _inputs()
    o_ref, f_ref = oracle.fwd(q, k, v, g, beta, init)
    for r in range(world):
        a, b = cuts[r], cuts[r + 1]
        np.testing.assert_allclose(res[r][0], o_ref[:, a:b], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res[r][1], f_ref, rtol=1e-10, atol=1e-12)
