"""GPU parity of the in-place decode step against the oracle, and decode ==
prefill consistency (T decode steps reproduce a T-token forward)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import oracle
import synth
from parity import assert_close, errors

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _oracle_state(state, sel=None):
    s = state if sel is None else state[sel]
    return s.detach().cpu().double().numpy().copy()


@pytest.mark.parametrize("dtype,dk,dv", [(torch.bfloat16, 128, 128), (torch.float32, 128, 128),
                                         (torch.float32, 16, 16), (torch.bfloat16, 64, 32),
                                         (torch.float32, 32, 128)])
def test_decode_steps_match_oracle(dtype, dk, dv):
    spec = synth.DecodeSpec("t", 3, 5, dk, dv, dtype, 21, 8)
    state = synth.make_decode_state(spec, DEV)
    ref = _oracle_state(state)
    for step in range(spec.steps):
        x = synth.make_decode_step(spec, step, DEV)
        out = kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
        o_ref = oracle.decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], ref)
        assert_close(out, o_ref, dtype, f"decode out step {step}")
    torch.cuda.synchronize()
    assert_close(state, ref, dtype, "decode state")


def test_decode_full_shape_sampled():
    """B=512, H=96, dk=dv=128, bf16: 3 steps; sequences/heads sampled for the oracle."""
    spec = synth.DECODE
    state = synth.make_decode_state(spec, DEV)
    bsel = torch.tensor([0, 1, 255, 511])
    hsel = torch.tensor([0, 47, 95])
    ref = state[bsel][:, hsel].cpu().double().numpy().copy()
    for step in range(3):
        x = synth.make_decode_step(spec, step, DEV)
        out = kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
        pick = lambda t: t[bsel][:, hsel]
        o_ref = oracle.decode_step(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["g"]), pick(x["beta"]), ref)
        assert_close(pick(out), o_ref, torch.bfloat16, f"decode full out step {step}")
    torch.cuda.synchronize()
    assert_close(state[bsel][:, hsel], ref, torch.bfloat16, "decode full state")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_decode_equals_prefill(dtype):
    """T decode steps from S0 == one forward over the same T tokens."""
    B, H, T = 2, 4, 96
    spec = synth.PrefillSpec("dp", B, T, H, 128, 128, dtype, 31, init=True)
    inp = synth.make_prefill(spec, DEV)
    o_pre, f_pre = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"])
    state = inp["init_state"].clone()
    outs = []
    for t in range(T):
        sl = lambda x: x[:, t].contiguous()
        outs.append(kda.kda_decode_step(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["g"]), sl(inp["beta"]),
                                        state))
    o_dec = torch.stack(outs, 1)
    torch.cuda.synchronize()
    o_ref, f_ref = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"])
    assert_close(o_dec, o_ref, dtype, "decode path")
    assert_close(state, f_ref, dtype, "decode final")
    assert_close(o_pre, o_ref, dtype, "prefill path")
    tol = 1e-2 if dtype == torch.bfloat16 else 1e-4
    assert errors(o_dec, o_pre)["rel_fro"] < tol
    assert errors(state, f_pre)["rel_fro"] < tol
