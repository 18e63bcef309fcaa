"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Sizes span several 64-token chunks and ragged
tails; the full-size workloads are checked on sampled heads."""
import numpy as np
import pytest
import torch

import gated_delta_rule_121_b200 as kda
import oracle
import synth
from parity import ErrorAccumulator, assert_close, errors

pytestmark = pytest.mark.gpu
DEV = "cuda"


def run_gpu(inp):
    return kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"],
                       inp["cu_seqlens"])


def run_oracle(inp, heads=None):
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    init = inp["init_state"]
    if init is not None and heads is not None:
        init = init[:, heads]
    return oracle.fwd(sel(inp["q"]), sel(inp["k"]), sel(inp["v"]), sel(inp["g"]), sel(inp["beta"]), init,
                      inp["cu_seqlens"])


def check(inp, dtype, heads=None, what="", literal=True):
    out, fin = run_gpu(inp)
    torch.cuda.synchronize()
    if heads is not None:
        return check_sampled(inp, out, fin, dtype, heads, what)
    o_ref, f_ref = run_oracle(inp, heads)
    eo = assert_close(out, o_ref, dtype, f"{what} out", literal=literal)
    ef = assert_close(fin, f_ref, dtype, f"{what} final_state", literal=literal)
    return eo, ef


def check_sampled(inp, out, fin, dtype, heads, what, per_call=2):
    """The oracle on the sampled heads, a few at a time, with the errors
    accumulated over all of them (literal bounds)."""
    ao, af = ErrorAccumulator(dtype, f"{what} out"), ErrorAccumulator(dtype, f"{what} final_state")
    for i in range(0, len(heads), per_call):
        hs = list(heads[i:i + per_call])
        o_ref, f_ref = run_oracle(inp, hs)
        ao.add(out[:, :, hs], o_ref)
        af.add(fin[:, hs], f_ref)
        del o_ref, f_ref
    return ao.check(), af.check()


def sampled_heads(H, n=8, seed=0):
    """n seeded heads, always including the first and the last."""
    rest = np.random.default_rng(seed).choice(np.arange(1, H - 1), size=n - 2, replace=False)
    return sorted({0, H - 1, *rest.tolist()})


def test_tiny_fp32_exact_path():
    inp = synth.make_prefill(synth.TINY, DEV)
    check(inp, torch.float32, what="tiny fp32")


@pytest.mark.parametrize("T", [64, 100, 257])
def test_bf16_small_ragged(T):
    inp = synth.make_prefill(synth.MID, DEV, T=T, B=2, H=3)
    check(inp, torch.bfloat16, what=f"bf16 T={T}")


def test_mid_prefill_full():
    inp = synth.make_prefill(synth.MID, DEV)
    eo, ef = check(inp, torch.bfloat16, what="mid B2 H16 T4096")
    print("mid errors", eo, ef)


def test_mid_prefill_fp32():
    """The mid shape with fp32 q/k/v (the CUDA-core path) at the 1e-4 bar."""
    spec = synth.PrefillSpec("mid_fp32", 2, 4096, 16, 128, 128, torch.float32, 13, init=True)
    inp = synth.make_prefill(spec, DEV)
    eo, ef = check(inp, torch.float32, what="mid fp32")
    print("mid fp32 errors", eo, ef)


def test_stress_model_range_decay():
    """g = -5 sigmoid(z): chunk totals far below the factorisation floor."""
    inp = synth.make_prefill(synth.STRESS, DEV)
    assert float(inp["g"].min()) < -4.0
    check(inp, torch.bfloat16, what="stress g>=-5", literal=False)


def test_mixed_decay_chunks():
    """Alternate mild and model-range decay so both Gram paths meet in one chain."""
    inp = synth.make_prefill(synth.MID, DEV, T=512, B=1, H=2)
    g = inp["g"].clone()
    for c in range(0, 512, 128):
        g[:, c:c + 64] *= 64.0          # -5 * sigmoid(z) on every other chunk
    inp["g"] = g.contiguous()
    check(inp, torch.bfloat16, what="mixed decay", literal=False)


def test_model_range_decay_ragged_packed():
    """Strongly decaying chunks (level Gram) that end mid-chunk: packed
    sequences of ragged lengths with g = -5 sigmoid(z), each with its own
    initial state."""
    inp = synth.make_prefill(synth.VARLEN, DEV, H=3, lengths=[1, 37, 64, 100, 130, 0, 257])
    inp["g"] = (inp["g"] * 64.0).contiguous()
    assert float(inp["g"].min()) < -4.0
    check(inp, torch.bfloat16, what="varlen model-range decay", literal=False)


def test_decay_beyond_the_model_bound():
    """g = -20 sigmoid(z), four times past the model's bound g >= -5: every
    factor of the strongly decaying path stays at most 1 for any g <= 0."""
    inp = synth.make_prefill(synth.VARLEN, DEV, H=2, lengths=[257, 64, 3, 190])
    inp["g"] = (inp["g"] * 256.0).contiguous()
    assert float(inp["g"].min()) < -15.0
    check(inp, torch.bfloat16, what="g >= -20", literal=False)


@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 130, 0, 200], [0], [5], [300, 0, 0, 64]])
def test_varlen_ragged_and_empty(lengths):
    inp = synth.make_prefill(synth.VARLEN, DEV, H=4, lengths=lengths)
    check(inp, torch.bfloat16, what=f"varlen {lengths}")


def test_varlen_fp32_small_dims():
    spec = synth.PrefillSpec("v32", 1, 0, 3, 32, 64, torch.float32, 11, init=True)
    inp = synth.make_prefill(spec, DEV, lengths=[17, 0, 64, 90])
    check(inp, torch.float32, what="fp32 dk32 dv64 varlen")


@pytest.mark.parametrize("dk,dv", [(16, 16), (64, 128), (128, 32), (64, 64)])
def test_bf16_other_dims(dk, dv):
    spec = synth.PrefillSpec("dims", 2, 0, 2, dk, dv, torch.bfloat16, 12, init=True)
    inp = synth.make_prefill(spec, DEV, T=150)
    check(inp, torch.bfloat16, what=f"bf16 dk{dk} dv{dv}")


def test_final_state_may_alias_init_state():
    """In-place chaining: final_state given as the init_state tensor itself."""
    inp = synth.make_prefill(synth.MID, DEV, T=300, B=2, H=3)
    ref_out, ref_fin = run_gpu(inp)
    state = inp["init_state"].clone()
    out, fin = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], state, None, final_state=state)
    torch.cuda.synchronize()
    assert fin.data_ptr() == state.data_ptr()
    assert torch.equal(out, ref_out) and torch.equal(fin, ref_fin)


def test_many_short_packed_sequences():
    """200 packed sequences of 0..300 tokens: partial chunks everywhere and the
    longest-first order over many length buckets."""
    g = torch.Generator().manual_seed(77)
    lengths = torch.randint(0, 301, (200,), generator=g).tolist()
    lengths[3] = 0
    lengths[7] = 1
    inp = synth.make_prefill(synth.VARLEN, DEV, H=2, lengths=lengths)
    check(inp, torch.bfloat16, what="200 short packed sequences")


def test_batched_zero_tokens_returns_init_state():
    inp = synth.make_prefill(synth.MID, DEV, T=64, B=2, H=2)
    e = lambda t: t[:, :0].contiguous()
    out, fin = kda.kda_fwd(e(inp["q"]), e(inp["k"]), e(inp["v"]), e(inp["g"]), e(inp["beta"]), inp["init_state"])
    torch.cuda.synchronize()
    assert out.shape[1] == 0
    assert torch.equal(fin, inp["init_state"])


def test_no_final_state_and_zero_init():
    inp = synth.make_prefill(synth.MID, DEV, T=200, B=1, H=2)
    out, fin = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None, None,
                           output_final_state=False)
    assert fin is None
    o_ref, _ = oracle.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], None)
    assert_close(out, o_ref, torch.bfloat16, "zero init")


def test_chained_calls_equal_single_call():
    """Chunked-prefill resume: [0,T1) then [T1,T) from the returned state."""
    inp = synth.make_prefill(synth.MID, DEV, T=640, B=1, H=4)
    o_full, f_full = run_gpu(inp)
    T1 = 320
    part = lambda t, s: t[:, s].contiguous()
    a = {k: (part(v, slice(0, T1)) if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    o1, mid = run_gpu(a)
    b = {k: (part(v, slice(T1, None)) if k in ("q", "k", "v", "g", "beta") else v) for k, v in inp.items()}
    b["init_state"] = mid
    o2, f2 = run_gpu(b)
    torch.cuda.synchronize()
    o_ref, f_ref = run_oracle(inp)
    assert_close(torch.cat([o1, o2], 1), o_ref, torch.bfloat16, "chained out")
    assert_close(f2, f_ref, torch.bfloat16, "chained final_state")
    assert_close(o_full, o_ref, torch.bfloat16, "single-call out")
    # the two GPU paths agree with each other far inside the oracle tolerance
    assert errors(torch.cat([o1, o2], 1), o_full)["rel_fro"] < 5e-3
    assert errors(f2, f_full)["rel_fro"] < 5e-3


def test_model_shaped_prefill_sampled_heads():
    """B=1, H=96, T=65536 (the 64K pretraining shape), eight seeded heads
    including 0 and 95, at the literal max-abs bound."""
    inp = synth.make_prefill(synth.PRETRAIN, DEV)
    eo, ef = check(inp, torch.bfloat16, heads=sampled_heads(96, seed=2), what="prefill H96 T65536")
    print("pretrain errors", eo, ef)


def test_packed_varlen_full_size_sampled_heads():
    """The packed long-context workload at full size: H=32, 1,048,576 tokens in
    sequences of log-uniform length in [1024, 262144], each with its own
    initial state; eight seeded heads (0 and 31 among them) of every sequence
    checked at the literal max-abs bound."""
    inp = synth.make_prefill(synth.VARLEN, DEV)
    cu = inp["cu_seqlens"].cpu()
    assert int(cu[-1]) == 1 << 20 and cu.numel() - 1 >= 3
    eo, ef = check(inp, torch.bfloat16, heads=sampled_heads(32, seed=3), what="varlen H32 T1M")
    print("varlen errors", cu.numel() - 1, "sequences", eo, ef)


@pytest.mark.parametrize("decay", ["mild", "model_range"])
def test_debug_intermediates_match_chunk_model(decay):
    """One chunk's P, A, T', W', U, Δ, O and S against the fp64 chunk model:
    with mild decay the chunk takes the end-referenced Gram, with model-range
    decay (g down to -5) the level Gram and start-referenced operands."""
    from chunk_model import chunk_forward
    inp = synth.make_prefill(synth.MID, DEV, T=64, B=1, H=1)
    if decay == "model_range":
        inp["g"] = (inp["g"] * 64.0).contiguous()  # -5 sigmoid(z)
        assert float(inp["g"].sum(1).min()) < -7.0  # chunk total below the end-referenced floor
    dbg = torch.zeros(kda.lib().kda_testing_debug_floats(), dtype=torch.float32, device=DEV)
    out, fin = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], _debug=dbg)
    torch.cuda.synchronize()
    f = lambda t: t[0, :, 0].cpu().double().numpy()
    O, S, it = chunk_forward(f(inp["q"]), f(inp["k"]), f(inp["v"]), f(inp["g"]), f(inp["beta"]),
                             inp["init_state"][0, 0].cpu().double().numpy(), C=64, keep=True)
    d = dbg.cpu().double().numpy()
    it = it[0]
    checks = [("P", d[0:4096].reshape(64, 64), it["P"]),
              ("A", d[4096:8192].reshape(64, 64), it["A"]),
              ("T'", d[8192:12288].reshape(64, 64), it["T"] * f(inp["beta"])[None, :]),
              # fast chunks store W' = W Diag(exp(-G_C)) (operands referenced to the chunk
              # end), general chunks W' = W (referenced to the chunk start)
              ("W'", d[12288:20480].reshape(64, 128),
               it["W"] * (np.exp(-it["G"][-1])[None, :] if decay == "mild" else 1.0)),
              ("U", d[20480:28672].reshape(64, 128), it["U"]),
              ("Delta", d[28672:36864].reshape(64, 128), it["Delta"]),
              ("O", d[36864:45056].reshape(64, 128), O),
              ("S", d[45056:61440].reshape(128, 128), S),
              ("G_C", d[61440:61568], it["G"][-1])]
    bad = []
    for name, got, ref in checks:
        e = errors(got, ref)
        if not e["rel_fro"] < 2e-2:
            bad.append((name, e))
    assert not bad, bad


def test_timeout_path_reports_status_and_context_survives():
    """A wait on a barrier nothing signals gives up after 1 ms, the status
    word says so, and the next call on the same context succeeds."""
    inp = synth.make_prefill(synth.MID, DEV, T=256, B=1, H=2)
    ws = kda.alloc_workspace(1, 256, 2, 128, 128)
    kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], workspace=ws,
                _wait_ns=1_000_000, _inject_stuck=True)
    assert kda.kda_workspace_status(ws) == kda.KDA_ERR_TIMEOUT
    # the context is still usable and a normal call succeeds
    out, fin = kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"],
                           workspace=ws)
    assert kda.kda_workspace_status(ws) == kda.KDA_OK
    o_ref, f_ref = run_oracle(inp)
    assert_close(out, o_ref, torch.bfloat16, "after timeout")


@pytest.mark.parametrize("what", ["v", "state"])
def test_fp16_range_overflow_is_reported(what):
    """Values beyond the fp16 range of the tensor-core operands (a huge v, or
    a huge initial state) are reported as KDA_ERR_RANGE in the status word;
    the next call on the same workspace starts clean."""
    inp = synth.make_prefill(synth.MID, DEV, T=192, B=1, H=2)
    ws = kda.alloc_workspace(1, 192, 2, 128, 128)
    args = {k: v for k, v in inp.items()}
    if what == "v":
        args["v"] = (inp["v"].float() * 1e6).to(torch.bfloat16)
    else:
        args["init_state"] = inp["init_state"] * 1e9
    kda.kda_fwd(args["q"], args["k"], args["v"], args["g"], args["beta"], args["init_state"], workspace=ws)
    assert kda.kda_workspace_status(ws) == kda.KDA_ERR_RANGE
    kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], workspace=ws)
    assert kda.kda_workspace_status(ws) == kda.KDA_OK


@pytest.mark.parametrize("case", ["batched_b2", "batched_b11", "one_sequence_sliced", "one_sequence_short",
                                  "packed", "batched_unaligned_beta", "one_sequence_no_final_state"])
def test_host_buffer_entry_point_matches_device_call(case):
    """kda_fwd_host (host buffers, copies enqueued by the library) returns the
    bits kda_fwd returns on device buffers: in one piece (packed batches), in
    pieces of whole sequences overlapping copies and compute (B > 1: 2 and 11
    pieces), and in token slices of one sequence carried through the final
    state (B = 1, 1000 tokens: 16 slices starting on chunk boundaries, the last
    ragged), called twice on the same buffers; in one piece where a piece's
    beta rows would not start on 16 bytes (T H = 303) and for one sequence
    without a final-state buffer."""
    if case == "packed":
        inp = synth.make_prefill(synth.VARLEN, DEV, H=3, lengths=[70, 0, 129])
    elif case == "batched_b2":
        inp = synth.make_prefill(synth.MID, DEV, T=200, B=2, H=3)
    elif case == "batched_b11":
        inp = synth.make_prefill(synth.MID, DEV, T=130, B=11, H=2)
    elif case == "one_sequence_sliced":
        inp = synth.make_prefill(synth.MID, DEV, T=1000, B=1, H=3)
    elif case == "batched_unaligned_beta":
        inp = synth.make_prefill(synth.MID, DEV, T=101, B=3, H=3)
    elif case == "one_sequence_no_final_state":
        inp = synth.make_prefill(synth.MID, DEV, T=700, B=1, H=2)
    else:
        inp = synth.make_prefill(synth.PRETRAIN, DEV, T=100, B=1, H=2)  # no initial state, 2 slices
    ref_out, ref_fin = run_gpu(inp)
    host = {n: (None if t is None else t.cpu().pin_memory()) for n, t in inp.items()}
    bufs = None
    want_final = case != "one_sequence_no_final_state"
    for _ in range(2):
        out_h, fin_h, bufs = kda.kda_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"],
                                              host["init_state"], host["cu_seqlens"], device=DEV, dev_buffers=bufs,
                                              output_final_state=want_final)
        torch.cuda.synchronize()
        assert torch.equal(out_h, ref_out.cpu())
        assert (fin_h is None) if not want_final else torch.equal(fin_h, ref_fin.cpu())
