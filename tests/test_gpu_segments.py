"""GPU parity of the segment decomposition (intra-device context parallelism,
KCP pieces) and of the interval checkpoints, through the C ABI, against the
fp64 oracle: zero-start outputs and states, transitions and transformed
queries (oracle.transition), the prefix composition and the output
correction (their definitions in fp64), whole forwards split into segments
whose boundaries fall inside 64-token chunks, and checkpoint states (the
oracle's final state over each prefix)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import oracle
import synth
from parity import ErrorAccumulator, assert_close, errors

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _args(inp):
    return inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"]


SEG_CASES = {
    "bf16_batched_tc": lambda: synth.make_prefill(synth.MID, DEV, T=300, B=2, H=3),
    "bf16_packed_tc": lambda: synth.make_prefill(synth.VARLEN, DEV, H=3, lengths=[130, 0, 1, 64, 257]),
    "bf16_model_range_tc": lambda: _scaled_g(synth.make_prefill(synth.MID, DEV, T=200, B=1, H=2), 64.0),
    "fp32_packed_simt": lambda: synth.make_prefill(synth.PrefillSpec("s32", 1, 0, 3, 32, 32, torch.float32, 41),
                                                   DEV, lengths=[40, 0, 77]),
    "bf16_d64_simt": lambda: synth.make_prefill(synth.PrefillSpec("s64", 2, 0, 2, 64, 64, torch.bfloat16, 42),
                                                DEV, T=90),
}


def _scaled_g(inp, f):
    inp["g"] = (inp["g"] * f).contiguous()
    return inp


@pytest.mark.parametrize("case", sorted(SEG_CASES))
def test_segment_pieces_match_oracle(case):
    inp = SEG_CASES[case]()
    dtype = inp["q"].dtype
    literal = case != "bf16_model_range_tc"
    cu = inp["cu_seqlens"]
    o0, s0, qh, M = kda.kda_segment_fwd(*_args(inp), cu_seqlens=cu)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.fwd(*_args(inp), None, cu)
    qh_ref, M_ref = oracle.transition(inp["q"], inp["k"], inp["g"], inp["beta"], cu)
    assert_close(o0, o_ref, dtype, f"{case} zero-start out", literal=literal)
    assert_close(s0, s_ref, dtype, f"{case} zero-start state", literal=literal)
    assert_close(qh, qh_ref, dtype, f"{case} qhat", literal=literal)
    # The transition is dimensionless with the identity as its scale: it acts
    # on an incoming state, so its error is measured per (sequence, head)
    # against max(|M|_F, 1e-2) (a strongly decaying segment's M is ~0).
    Mg, Mr = M.double().cpu().numpy(), np.asarray(M_ref)
    err = np.linalg.norm((Mg - Mr).reshape(Mr.shape[0], Mr.shape[1], -1), axis=-1)
    scale = np.maximum(np.linalg.norm(Mr.reshape(Mr.shape[0], Mr.shape[1], -1), axis=-1), 1e-2)
    tol = 1e-4 if dtype == torch.float32 else 5e-3
    assert (err / scale).max() <= tol, f"{case} transition: {(err / scale).max():.3e}"


def _compose_ref(M, S0, init, R, rank_major):
    M, S0 = M.double().cpu().numpy(), S0.double().cpu().numpy()
    P, H, dk, dv = S0.shape
    N = P // R
    idx = (lambda m, r: r * N + m) if rank_major else (lambda m, r: m * R + r)
    s_in = np.zeros_like(S0)
    fin = np.zeros((N, H, dk, dv))
    for m in range(N):
        cur = init[m].double().cpu().numpy() if init is not None else np.zeros((H, dk, dv))
        for r in range(R):
            p = idx(m, r)
            s_in[p] = cur
            cur = S0[p] + M[p] @ cur
        fin[m] = cur
    return s_in, fin


@pytest.mark.parametrize("d,rank_major,with_init", [(128, False, True), (128, True, True), (32, False, False),
                                                    (64, True, False)])
def test_state_compose_matches_definition(d, rank_major, with_init):
    g = torch.Generator(device=DEV).manual_seed(d)
    R, N, H = 3, 2, 2
    M = (torch.randn((R * N, H, d, d), generator=g, device=DEV) / d ** 0.5).contiguous()
    S0 = torch.randn((R * N, H, d, d), generator=g, device=DEV)
    init = torch.randn((N, H, d, d), generator=g, device=DEV) if with_init else None
    s_in, fin = kda.kda_state_compose(M, S0, R, init_state=init, rank_major=rank_major)
    torch.cuda.synchronize()
    s_ref, f_ref = _compose_ref(M, S0, init, R, rank_major)
    assert errors(s_in, s_ref)["rel_fro"] < 1e-5
    assert errors(fin, f_ref)["rel_fro"] < 1e-5


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("lengths", [None, [5, 0, 64, 150, 1, 100]])
def test_output_correct_matches_definition(dtype, lengths):
    g = torch.Generator(device=DEV).manual_seed(7)
    H, dk, dv = 2, 128, 128
    if lengths is None:
        B, T, N, cu = 2, 200, 2, None
    else:
        B, T, N = 1, sum(lengths), len(lengths)
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device=DEV)
    o0 = torch.randn((B, T, H, dv), generator=g, device=DEV)
    qh = torch.randn((B, T, H, dk), generator=g, device=DEV) * 0.3
    s_in = torch.randn((N, H, dk, dv), generator=g, device=DEV) * 0.2
    out = kda.kda_output_correct(o0, qh, s_in, cu_seqlens=cu, dtype=dtype)
    torch.cuda.synchronize()
    o0n, qhn, sn = (x.double().cpu().numpy() for x in (o0, qh, s_in))
    seq = np.repeat(np.arange(N), lengths) if lengths is not None else np.repeat(np.arange(B), T)
    ref = o0n.reshape(-1, H, dv) + np.einsum("thi,thij->thj", qhn.reshape(-1, H, dk), sn[seq])
    ref = ref.reshape(B, T, H, dv)
    if dtype == torch.bfloat16:
        assert_close(out, ref, dtype, "correct bf16")
    else:
        assert errors(out, ref)["rel_fro"] < 1e-6


CP_CASES = {
    "mid_nseg2": (lambda: synth.make_prefill(synth.MID, DEV), 2, True),
    "mid_nseg3": (lambda: synth.make_prefill(synth.MID, DEV), 3, True),
    "t65536_nseg7": (lambda: synth.make_prefill(synth.PRETRAIN, DEV, H=2), 7, True),
    "packed_ragged_nseg3": (lambda: synth.make_prefill(synth.VARLEN, DEV, H=3, lengths=[1, 63, 0, 700, 130]), 3,
                            True),
    "stress_nseg2": (lambda: synth.make_prefill(synth.STRESS, DEV, H=4), 2, False),
    "fp32_d32_nseg4": (lambda: synth.make_prefill(synth.PrefillSpec("cp32", 2, 0, 3, 32, 32, torch.float32, 43,
                                                                    init=True), DEV, T=333), 4, True),
}


@pytest.mark.parametrize("case", sorted(CP_CASES))
def test_fwd_cp_matches_oracle(case):
    make, n_seg, literal = CP_CASES[case]
    inp = make()
    dtype = inp["q"].dtype
    out, fin = kda.kda_fwd_cp(*_args(inp), inp["init_state"], inp["cu_seqlens"], n_seg=n_seg)
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.fwd(*_args(inp), inp["init_state"], inp["cu_seqlens"])
    eo = assert_close(out, o_ref, dtype, f"{case} out", literal=literal)
    ef = assert_close(fin, f_ref, dtype, f"{case} final_state", literal=literal)
    print(case, eo, ef)


def test_fwd_cp_segment_boundaries_fall_inside_chunks():
    """The T=65536 split into 7 segments puts every cut off the 64-token grid."""
    T, R = 65536, 7
    cuts = [(T * r) // R for r in range(1, R)]
    assert all(c % 64 for c in cuts)


def test_cp_segments_planner():
    sm = torch.cuda.get_device_properties(0).multi_processor_count
    assert kda.kda_cp_segments(2, 4096, 16, sm) >= 2              # the mid batch: 32 chains of 4096 tokens
    assert kda.kda_cp_segments(1, 65536, 96, sm) == 1             # 96 chains already fill the device
    assert kda.kda_cp_segments(1, 256, 4, sm) == 1                # too short to split


def test_kcp_ranks_emulated_on_one_device():
    """The KCP data path of three ranks, run one after another on this device
    (the all-gather replaced by stacking the ranks' pieces): each rank's
    outputs and the final state against the oracle on the whole sequence."""
    from gated_delta_rule_121_b200 import kcp
    inp = synth.make_prefill(synth.MID, DEV, T=3000, B=2, H=4)
    cuts = [0, 1100, 1101, 3000]
    R = len(cuts) - 1
    pieces = []
    for r in range(R):
        sl = lambda t: t[:, cuts[r]:cuts[r + 1]].contiguous()
        pieces.append(kcp.kcp_pieces(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"])))
    trans = torch.cat([p[2] for p in pieces], 0)
    s_zero = torch.cat([p[3] for p in pieces], 0)
    state_in, fin = kcp.kcp_combine(trans, s_zero, R, inp["init_state"])
    B = 2
    outs = [kcp.kcp_finish(pieces[r][0], pieces[r][1], state_in[r * B:(r + 1) * B].contiguous(), torch.bfloat16)
            for r in range(R)]
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.fwd(*_args(inp), inp["init_state"])
    assert_close(torch.cat(outs, 1), o_ref, torch.bfloat16, "kcp out")
    assert_close(fin, f_ref, torch.bfloat16, "kcp final_state")


CKPT_CASES = {
    "bf16_batched_tc": (lambda: synth.make_prefill(synth.MID, DEV, T=1000, B=2, H=3), 128),
    "bf16_packed_tc": (lambda: synth.make_prefill(synth.VARLEN, DEV, H=2, lengths=[0, 64, 511, 512, 1030, 129]),
                       256),
    "bf16_packed_512": (lambda: synth.make_prefill(synth.VARLEN, DEV, H=2, lengths=[2600, 512, 100]), 512),
    "fp32_packed_simt": (lambda: synth.make_prefill(synth.PrefillSpec("c32", 1, 0, 2, 32, 64, torch.float32, 44,
                                                                      init=True), DEV, lengths=[70, 200, 0, 64]),
                         64),
}


def _seq_bounds(inp):
    if inp["cu_seqlens"] is not None:
        cu = inp["cu_seqlens"].cpu().tolist()
        return [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    B, T = inp["q"].shape[:2]
    return [(b, 0, T) for b in range(B)]


@pytest.mark.parametrize("case", sorted(CKPT_CASES))
def test_checkpoints_match_oracle_prefix_states(case):
    make, interval = CKPT_CASES[case]
    inp = make()
    dtype = inp["q"].dtype
    args = (*_args(inp), inp["init_state"], inp["cu_seqlens"])
    out, fin, ck = kda.kda_fwd_checkpoints(*args, interval=interval)
    ref_out, ref_fin = kda.kda_fwd(*args)
    torch.cuda.synchronize()
    # the forward itself is unchanged by the checkpoint writes
    assert torch.equal(out, ref_out) and torch.equal(fin, ref_fin)
    slot = 0
    acc = ErrorAccumulator(dtype, f"{case} checkpoints")
    init = inp["init_state"]
    for n, (b, a, e) in enumerate(_seq_bounds(inp)):
        for m in range(1, (e - a) // interval + 1):
            p = a + m * interval
            sl = lambda t: t[b:b + 1, a:p].contiguous()
            s0 = None if init is None else init[n:n + 1]
            _, s_ref = oracle.fwd(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]), s0)
            acc.add(ck[slot], s_ref[0])
            slot += 1
    assert slot == ck.shape[0]
    if slot:
        acc.check()


def test_checkpoint_capacity_overflow_is_reported():
    inp = synth.make_prefill(synth.VARLEN, DEV, H=2, lengths=[300, 700])
    ws = torch.empty(kda.lib().kda_fwd_checkpoints_workspace_size(2, 1000, 2, 128, 128, kda.KDA_BF16),
                     dtype=torch.uint8, device=DEV)
    kda.kda_fwd_checkpoints(*_args(inp), None, inp["cu_seqlens"], interval=128, capacity=3, workspace=ws)
    assert kda.kda_workspace_status(ws) == kda.KDA_ERR_INVALID_ARG
