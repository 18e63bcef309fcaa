"""GPU parity of the decode paths added to the single-token step: the fused
input prologue (q, k normalised and the bounded gate applied in the kernel)
and speculative verification with state replay, through the C ABI against
the oracle (oracle.decode_step_gated, oracle.spec_decode)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import oracle
import synth
from parity import ErrorAccumulator, assert_close

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype,dk,dv", [(torch.bfloat16, 128, 128), (torch.float32, 64, 32)])
@pytest.mark.parametrize("z_shift", [-5.0, 0.0])
def test_gated_decode_steps_match_oracle(dtype, dk, dv, z_shift):
    spec = synth.DecodeSpec("gd", 3, 4, dk, dv, dtype, 51, 6)
    state = synth.make_decode_state(spec, DEV)
    ref = state.double().cpu().numpy().copy()
    A_log = torch.tensor([0.2, -0.3, 0.0, 0.5], device=DEV)
    literal = z_shift < -1
    for step in range(spec.steps):
        x = synth.make_spec_window(spec, step, 1, DEV, prologue=True, z_shift=z_shift)
        one = {n: t[:, 0].contiguous() for n, t in x.items()}
        out = kda.kda_decode_step_gated(one["q"], one["k"], one["v"], one["g"], A_log, one["beta"], state)
        o_ref = oracle.decode_step_gated(one["q"], one["k"], one["v"], one["g"], A_log.cpu(), one["beta"], ref)
        assert_close(out, o_ref, dtype, f"gated decode out step {step}", literal=literal)
    torch.cuda.synchronize()
    assert_close(state, ref, dtype, "gated decode state", literal=literal)


def _spec_case(dtype, dk, dv, B, H, Wp, W, seed, prologue, steps):
    spec = synth.DecodeSpec("sp", B, H, dk, dv, dtype, seed, steps)
    state = synth.make_decode_state(spec, DEV)
    ref = state.double().cpu().numpy().copy()
    A_log = (torch.randn(H, generator=torch.Generator().manual_seed(seed)) * 0.5).to(DEV) if prologue else None
    gen = np.random.default_rng(seed)
    prev = None
    outs = []
    for step in range(steps):
        cur = synth.make_spec_window(spec, step, W, DEV, prologue=prologue)
        na = torch.tensor(gen.integers(0, Wp + 1, B), dtype=torch.int32, device=DEV) if prev is not None else None
        out = kda.kda_decode_spec(prev, na, cur, state, A_log=A_log)
        if prologue:
            conv = lambda d: None if d is None else dict(q=oracle.l2norm(d["q"]), k=oracle.l2norm(d["k"]), v=d["v"],
                                                         g=oracle.gate(d["g"], A_log.cpu()), beta=d["beta"])
            o_ref = oracle.spec_decode(conv(prev), None if na is None else na.cpu(), conv(cur), ref)
        else:
            o_ref = oracle.spec_decode(prev, None if na is None else na.cpu(), cur, ref)
        outs.append((out, o_ref))
        prev = cur
        Wp = W
    torch.cuda.synchronize()
    return state, ref, outs


@pytest.mark.parametrize("dtype,dk,dv", [(torch.bfloat16, 128, 128), (torch.float32, 32, 64),
                                         (torch.bfloat16, 64, 16)])
@pytest.mark.parametrize("W", [1, 4, 8])
@pytest.mark.parametrize("prologue", [False, True])
def test_spec_decode_matches_oracle(dtype, dk, dv, W, prologue):
    state, ref, outs = _spec_case(dtype, dk, dv, B=5, H=3, Wp=W, W=W, seed=61 + W, prologue=prologue, steps=5)
    for i, (o, r) in enumerate(outs):
        assert_close(o, r, dtype, f"spec out step {i}")
    assert_close(state, ref, dtype, "spec committed state")


@pytest.mark.parametrize("dtype,dk,dv", [(torch.bfloat16, 128, 128), (torch.float32, 16, 16),
                                         (torch.bfloat16, 128, 16)])
def test_spec_decode_longest_chunk(dtype, dk, dv):
    """Every draft of an 8-token window accepted, then a new 8-token window:
    chunks of the maximum 16 tokens (both 8-token halves of the pair sums)."""
    spec = synth.DecodeSpec("sp16", 3, 2, dk, dv, dtype, 83, 2)
    state = synth.make_decode_state(spec, DEV)
    ref = state.double().cpu().numpy().copy()
    prev = synth.make_spec_window(spec, 0, 8, DEV)
    out0 = kda.kda_decode_spec(None, None, prev, state)
    o0 = oracle.spec_decode(None, None, prev, ref)
    na = torch.full((3,), 8, dtype=torch.int32, device=DEV)
    cur = synth.make_spec_window(spec, 1, 8, DEV)
    out1 = kda.kda_decode_spec(prev, na, cur, state)
    o1 = oracle.spec_decode(prev, na.cpu(), cur, ref)
    torch.cuda.synchronize()
    assert_close(out0, o0, dtype, "first window")
    assert_close(out1, o1, dtype, "16-token chunk")
    assert_close(state, ref, dtype, "state after the 16-token chunk")


def test_spec_decode_replay_only_and_full_accept():
    """W = 0 only replays the accepted drafts; accepting every draft with a
    one-token window equals plain decode steps over the same tokens."""
    spec = synth.DecodeSpec("sp0", 4, 2, 128, 128, torch.bfloat16, 71, 3)
    s0 = synth.make_decode_state(spec, DEV)
    prev = synth.make_spec_window(spec, 0, 3, DEV)
    empty = {n: t[:, :0].contiguous() for n, t in prev.items()}
    na = torch.tensor([0, 1, 2, 3], dtype=torch.int32, device=DEV)
    st = s0.clone()
    kda.kda_decode_spec(prev, na, empty, st)
    ref = s0.double().cpu().numpy().copy()
    oracle.spec_decode(prev, na.cpu(), empty, ref)
    torch.cuda.synchronize()
    assert_close(st, ref, torch.bfloat16, "replay only")
    # all three drafts accepted + a bonus token == four plain decode steps
    cur = synth.make_spec_window(spec, 1, 1, DEV)
    st2 = s0.clone()
    out = kda.kda_decode_spec(prev, torch.full((4,), 3, dtype=torch.int32, device=DEV), cur, st2)
    st3 = s0.clone()
    for t in range(3):
        kda.kda_decode_step(*(prev[n][:, t].contiguous() for n in ("q", "k", "v", "g", "beta")), st3)
    o3 = kda.kda_decode_step(*(cur[n][:, 0].contiguous() for n in ("q", "k", "v", "g", "beta")), st3)
    torch.cuda.synchronize()
    assert torch.allclose(out[:, 0].float(), o3.float(), rtol=1e-2, atol=1e-2)
    assert (st2 - st3).abs().max().item() < 1e-5 * max(1.0, st3.abs().max().item())


def test_spec_decode_full_shape_sampled():
    """B=512, H=96, d=128: windows of 4 (bonus + 3 drafts) over 6 steps with
    random accept counts; 24 (sequence, head) pairs followed by the oracle."""
    spec = synth.DECODE
    B, H, W = spec.B, spec.H, 4
    state = synth.make_decode_state(spec, DEV)
    bsel = torch.tensor([0, 3, 200, 511])
    hsel = torch.tensor([0, 17, 50, 70, 88, 95])
    pick = lambda t: t[bsel][:, :, hsel].contiguous() if t.dim() >= 3 else t[bsel][:, :, hsel]
    ref = state[bsel][:, hsel].double().cpu().numpy().copy()
    gen = np.random.default_rng(5)
    prev = None
    acc = ErrorAccumulator(torch.bfloat16, "spec full-shape outputs")
    for step in range(6):
        cur = synth.make_spec_window(spec, step, W, DEV)
        na = torch.tensor(gen.integers(0, W + 1, B), dtype=torch.int32, device=DEV) if prev is not None else None
        out = kda.kda_decode_spec(prev, na, cur, state)
        sub = lambda d: None if d is None else {n: (t[bsel][:, :, hsel] if t.dim() == 4 else t[bsel][:, :, hsel])
                                                 for n, t in d.items()}
        o_ref = oracle.spec_decode(sub(prev), None if na is None else na[bsel].cpu(), sub(cur), ref)
        o = out[bsel][:, :, hsel]
        assert_close(o, o_ref, torch.bfloat16, f"spec full out step {step}")
        acc.add(o, o_ref)
        prev = cur
    torch.cuda.synchronize()
    acc.check()
    assert_close(state[bsel][:, hsel], ref, torch.bfloat16, "spec full committed state")
