"""kda_fwd_noalloc: the prefill entry point for callers that cannot allocate
device memory.  Through the C ABI, two calls in a row must reproduce what
kda_fwd (with a caller workspace) returns on the same inputs: the same kernel
runs on the same inputs, so the results are bit-identical (kda_fwd itself is
checked against the oracle by the parity tests).  The file name sorts last so
a run that stops at the first failure has already run every other test."""
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import synth

pytestmark = pytest.mark.gpu


def _reference(inp):
    return kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"],
                       inp["cu_seqlens"])


@pytest.mark.parametrize("case", ["packed", "fixed"])
def test_noalloc_matches_kda_fwd_twice(case):
    if case == "packed":  # the order array in the fixed scratch is exercised
        inp = synth.make_prefill(synth.VARLEN, "cuda", H=4, lengths=[200, 0, 65, 130, 1])
    else:
        inp = synth.make_prefill(synth.MID, "cuda", T=300, B=2, H=3)
    ref_out, ref_fin = _reference(inp)
    for _ in range(2):
        out, fin = kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                                       inp["init_state"], inp["cu_seqlens"])
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out), "noalloc out differs from kda_fwd"
        assert torch.equal(fin, ref_fin), "noalloc final_state differs from kda_fwd"
        assert kda.kda_fwd_noalloc_status() == kda.KDA_OK


def test_noalloc_reports_device_errors_through_its_status_call():
    """A value beyond the fp16 range of the tensor-core operands is reported by
    kda_fwd_noalloc_status; the next clean call reads back KDA_OK."""
    inp = synth.make_prefill(synth.MID, "cuda", T=192, B=1, H=2)
    big_v = (inp["v"].float() * 1e6).to(torch.bfloat16)
    kda.kda_fwd_noalloc(inp["q"], inp["k"], big_v, inp["g"], inp["beta"], inp["init_state"])
    assert kda.kda_fwd_noalloc_status() == kda.KDA_ERR_RANGE
    kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"])
    assert kda.kda_fwd_noalloc_status() == kda.KDA_OK


def test_noalloc_rejects_too_many_sequences():
    n = 8193
    lengths = [1] * n
    inp = synth.make_prefill(synth.VARLEN, "cuda", H=1, lengths=lengths)
    with pytest.raises(kda.KdaError) as e:
        kda.kda_fwd_noalloc(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, inp["cu_seqlens"])
    assert e.value.code == kda.KDA_ERR_WORKSPACE
