"""GPU parity of the in-place decode step against the oracle, and decode ==
prefill consistency (T decode steps reproduce a T-token forward)."""
import numpy as np
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import oracle
import synth
from parity import ErrorAccumulator, assert_close, errors

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


def test_decode_full_shape_256_steps_sampled():
    """The decode workload as specified: B=512, H=96, dk=dv=128, bf16 inputs,
    256 consecutive in-place steps on the resident fp32 state.  24 (sequence,
    head) pairs are followed by the fp64 oracle: every step's output and the
    state after the last step, at the literal bounds."""
    spec = synth.DECODE
    assert spec.steps == 256
    state = synth.make_decode_state(spec, DEV)
    bsel = torch.tensor([0, 1, 137, 255, 384, 511])
    hsel = torch.tensor([0, 31, 64, 95])
    pick = lambda t: t[bsel][:, hsel]
    ref = pick(state).cpu().double().numpy().copy()
    acc = ErrorAccumulator(torch.bfloat16, "decode outputs over 256 steps")
    out = torch.empty((spec.B, spec.H, spec.dv), dtype=spec.dtype, device=DEV)
    for step in range(spec.steps):
        x = synth.make_decode_step(spec, step, DEV)
        kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, out=out)
        o_ref = oracle.decode_step(pick(x["q"]), pick(x["k"]), pick(x["v"]), pick(x["g"]), pick(x["beta"]), ref)
        o = pick(out)
        assert_close(o, o_ref, torch.bfloat16, f"decode full out step {step}")
        acc.add(o, o_ref)
    torch.cuda.synchronize()
    acc.check()
    e = assert_close(pick(state), ref, torch.bfloat16, "decode full state after 256 steps")
    print("decode 256 steps: final state", e)


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
