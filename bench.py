#!/usr/bin/env python
"""Benchmark of the KDA forward pass on B200 through the C ABI.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...      # the fp64 CPU oracle arm
    python bench.py --capture NAME            # a few launches of a small case, for ncu
    python bench.py --phases [--workload NAME] # per-phase cycles (test-hook build)
    python bench.py --chains 64,96,148        # time per chunk against concurrent chains

Default workload: the model-shaped prefill B=1, H=96, T=65536, dk=dv=128,
bf16 q/k/v/o with fp32 log-decay, beta and state (the 64K pretraining
context with the model's 96 heads).  One step = one kda_fwd over that batch.
The same run also times, each under its own key: the B=512, H=96
single-token decode ("decode": one kda_decode_step per step, state updated
in place; "decode_gated" on the raw prologue inputs), speculative
verification ("decode_spec": windows of 4 with replay, and the step time for
windows of 1, 2, 4 and 8), the same prefill end to end from pinned host
buffers through kda_fwd_host ("e2e"), and the other prefill workloads
("workloads": the mid batch B=2 H=16 T=4096 plain and through kda_fwd_cp,
one tensor-parallel rank's 4 heads of the 64K prefill plain and through
kda_fwd_cp, the packed 1M-token batch, the model-range decay cases, the 64K
prefill with 512-token checkpoints and with the fused prologue, and one rank's
compute of the 64K prefill split over 8 ranks by KCP).
Inputs are synthetic (seeded) and resident in HBM before the timed region;
workloads smaller than the 126 MB L2 (or close to it) get an L2 flush before
every timed launch, the others are far larger than L2.

Metric: Mtoken-heads/s = tokens x heads / time / 1e6, plus the fraction of
the HBM roofline (measured copy bandwidth from MEASURED_PEAKS.json).

Multi-GPU (torchrun): every rank runs its own copy of the workload (the
heads and sequences are independent chains, so no data-path collective);
per-GPU work is fixed ("weak" scaling) and the value counts all ranks' work
over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA fwd Mtoken-heads/s at H=96,d=128 (prefill & decode); % of roofline"
UNIT = "Mtoken-heads/s"
CHUNK = 64
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def prefill_bytes(tokens_heads, chains, dk, dv, io_bytes, with_init):
    """Algorithmic HBM bytes of one forward: q,k,v,o in the I/O dtype, fp32
    log-decay and beta, plus the fp32 final state (and initial state)."""
    per_th = io_bytes * (2 * dk + 2 * dv) + 4 * dk + 4
    return tokens_heads * per_th + chains * dk * dv * 4 * (2 if with_init else 1)


def prefill_flops(tokens_heads, dk, dv, C=CHUNK):
    """Chunk-method flops per token-head: state products (W S, Q S, K^T Delta)
    6 dk dv, intra-chunk Gram/WY/output work C (6 dk + 4 dv), solve C^2/3."""
    return tokens_heads * (6 * dk * dv + C * (6 * dk + 4 * dv) + C * C / 3)


def decode_bytes(B, H, dk, dv, io_bytes):
    return B * H * (2 * dk * dv * 4 + io_bytes * (2 * dk + 2 * dv) + 4 * dk + 4)


def source_sha(name):
    src = os.path.join(ROOT, "gated_delta_rule_121_b200", "csrc", name)
    return hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]


def read_kv(path):
    kv = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.strip().split("=", 1)
            kv[k.strip()] = v.strip()
    return kv


def scaled_traffic(profile, source, units, fixed_bytes):
    """DRAM bytes per launch of a kernel from a committed ncu capture of a
    smaller case of the same kernel, scaled to this launch: the capture's
    bytes beyond its fixed part (states) per unit (token-head or decoded
    head), times this launch's units, plus this launch's fixed part.  None when
    the capture is missing or the kernel source changed since it was taken."""
    p = os.path.join(ROOT, "profiles", profile)
    if not os.path.exists(p):
        return None
    kv = read_kv(p)
    if kv.get("kernel_source_sha256") != source_sha(source):
        return None
    try:
        measured = float(kv["dram_bytes_read"]) + float(kv["dram_bytes_write"])
        per_unit = (measured - float(kv["capture_fixed_bytes"])) / float(kv["capture_units"])
    except (KeyError, ValueError, ZeroDivisionError):
        return None
    return per_unit * units + fixed_bytes


class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid):
        self.uuid, self.proc, self.lines = uuid, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 7:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, v in zip(names, f[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def time_loop(fn, steps, warmup, stream, dist_ctx):
    import torch
    for _ in range(warmup):
        fn()
    dist_ctx.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        fn()
    t1.record(stream)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    return t0.elapsed_time(t1) / 1000.0


def time_loop_flushed(fn, steps, warmup, stream, dist_ctx, flush_bytes=256 << 20):
    """Device time of `steps` launches of fn, each after a write of a buffer
    twice the size of L2 (so no launch finds its inputs in L2); only the
    launches are inside the timed events."""
    import torch
    buf = torch.empty(flush_bytes, dtype=torch.uint8, device=torch.cuda.current_device())
    for _ in range(warmup):
        fn()
    dist_ctx.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for e0, e1 in ev:
            buf.fill_(1)
            e0.record(stream)
            fn()
            e1.record(stream)
    torch.cuda.synchronize()
    dist_ctx.barrier()
    del buf
    return sum(e0.elapsed_time(e1) for e0, e1 in ev) / 1000.0


class Dist:
    """One process per GPU (torchrun env).  The only collectives are the
    timing barrier and the reductions of the per-rank results: every rank
    runs its own independent chains, so the data path has no exchange."""

    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.device = "cpu"

    def init(self, backend, timeout_s=120):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
            self.pg = dist
            self.device = "cuda" if backend == "nccl" else "cpu"

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def _reduce(self, x, op):
        if self.pg is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        self.pg.all_reduce(t, op=op)
        return float(t.item())

    def max(self, x):
        return self._reduce(x, self.pg.ReduceOp.MAX if self.pg is not None else None)

    def sum(self, x):
        return self._reduce(x, self.pg.ReduceOp.SUM if self.pg is not None else None)

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def job_throughput(d, units, seconds):
    """Whole-job rate: the units every rank processed over the slowest
    rank's time (seconds is this rank's own device time)."""
    return d.sum(units) / d.max(seconds)


def workload_spec(name):
    import synth
    return {"prefill64k": synth.PRETRAIN, "mid": synth.MID, "varlen": synth.VARLEN,
            "stress": synth.STRESS, "tp4": synth.TP4, "prefill64k_model_range": synth.PRETRAIN_MODEL_RANGE}[name]


# ----------------------------------------------------------------- oracle arm
def oracle_sample(spec, budget_s, threads):
    """Oracle throughput on a bounded sample of the workload: the first H_s
    heads and T_s tokens of one sequence, sized to ~budget_s seconds."""
    import oracle
    import synth
    H_s = max(1, min(spec.H, threads))
    cal = synth.make_prefill(spec, "cpu", T=256, B=1, H=1, lengths=[256] if spec.varlen else None)
    t = time.perf_counter()
    oracle.fwd(cal["q"], cal["k"], cal["v"], cal["g"], cal["beta"], None, cal["cu_seqlens"], nthreads=1)
    per_tok = (time.perf_counter() - t) / 256
    par = min(threads, H_s)
    T_s = int(max(64, min(spec.T if not spec.varlen else 262144, budget_s * par / (H_s * per_tok))))
    inp = synth.make_prefill(spec, "cpu", T=T_s, B=1, H=H_s, lengths=[T_s] if spec.varlen else None)
    t = time.perf_counter()
    oracle.fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], inp["cu_seqlens"],
               nthreads=threads)
    el = time.perf_counter() - t
    return dict(value=H_s * T_s / el / 1e6, unit=UNIT, cores=min(threads, H_s), kind="oracle",
                sample=f"{H_s} heads x {T_s} tokens of one sequence ({spec.name}), fp64 C recurrence",
                seconds=el)


def run_reference(args, d):
    import oracle
    spec = workload_spec(args.workload)
    if d.rank != 0:
        return
    threads = oracle.default_threads()
    budget = max(1.0, min(8.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(spec, budget, threads)
    vals, secs = [], 0.0
    last = None
    for _ in range(args.steps):
        last = oracle_sample(spec, budget, threads)
        vals.append(last["value"])
        secs += last["seconds"]
    v = statistics.median(vals)
    cb = dict(last)
    cb["value"] = v
    cb.pop("seconds", None)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": spec.name, "sample": cb["sample"]},
            "cpu_baseline": cb, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------- native arm
# ncu captures that give the DRAM traffic of a full launch (scaled by units):
# (profile file, kernel source, unit) per kernel.
TRAFFIC_PROFILES = {
    "kda_fwd_tc_kernel": ("kda_fwd_tc_prefill_h96_t4096_traffic.txt", "kda_fwd_tc.cu"),
    "kda_decode_kernel": ("kda_decode_b64_h96_traffic.txt", "kda_decode.cu"),
    "kda_spec_kernel": ("kda_spec_b64_h96_w4_traffic.txt", "kda_spec.cu"),
}
FLUSH = {"mid": True, "stress": True, "prefill64k": False, "varlen": False, "tp4": False,
         "prefill64k_model_range": False}


def bench_prefill(name, d, dev, stream, peaks, kda, synth, steps, warmup, with_traffic=False, variant=None):
    """Time `steps` forward calls over one workload; returns its JSON object
    and the inputs (for the end-to-end leg).  variant: None (kda_fwd), "cp"
    (kda_fwd_cp, every sequence split over the SMs), "ckpt512" (kda_fwd_checkpoints,
    the state every 512 tokens) or "gated" (kda_fwd_gated on the raw prologue
    inputs)."""
    import torch
    spec = workload_spec(name)
    if variant == "gated":  # raw prologue inputs: unnormalised q, k and bf16 decay logits z (mild decay)
        inp = synth.make_prologue_prefill(spec, dev, a_std=0.0)
        inp["g"] = inp.pop("z")
    else:
        inp = synth.make_prefill(spec, dev)
    q, k, v, g, beta, init, cu = (inp[n] for n in ("q", "k", "v", "g", "beta", "init_state", "cu_seqlens"))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = cu.numel() - 1 if cu is not None else B
    th = B * T * H
    out = torch.empty_like(v)
    fin = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    ws = kda.alloc_workspace(N, B * T, H, dk, dv, q.dtype, dev)
    extra = {}
    launches = 2 if (cu is not None and N > 1) else 1  # packed batches: the order kernel, then the forward
    ckpt_bytes = 0
    if variant == "cp":
        n_seg = kda.kda_cp_segments(N, (B * T) // N, H)
        ws = kda.alloc_cp_workspace(N, B * T, H, dk, dv, n_seg, q.dtype, dev)
        extra["n_seg"] = n_seg
        launches = 6  # segment offsets, order, state pass, composition, order, forward

        def step():
            kda.kda_fwd_cp(q, k, v, g, beta, init, cu, n_seg=n_seg, out=out, final_state=fin, workspace=ws,
                           stream=stream)
    elif variant == "gated":
        A_log = inp["A_log"]

        def step():
            kda.kda_fwd_gated(q, k, v, g, A_log, beta, init, cu, out=out, final_state=fin, workspace=ws, stream=stream)
    elif variant == "ckpt512":
        cap = N * (T // 512) if cu is None else int(((cu[1:] - cu[:-1]).cpu() // 512).sum())
        ck = torch.empty((cap, H, dk, dv), dtype=torch.float32, device=dev)
        n = kda.lib().kda_fwd_checkpoints_workspace_size(N, B * T, H, dk, dv, kda._DT[q.dtype])
        ws = torch.empty(n, dtype=torch.uint8, device=dev)
        extra.update(interval=512, checkpoints=cap)
        ckpt_bytes = cap * H * dk * dv * 4
        launches += 1 if cu is not None else 0

        def step():
            kda.kda_fwd_checkpoints(q, k, v, g, beta, init, cu, interval=512, capacity=cap, out=out,
                                    final_state=fin, checkpoints=ck, workspace=ws, stream=stream)
    else:
        def step():
            kda.kda_fwd(q, k, v, g, beta, init, cu, out=out, final_state=fin, workspace=ws, stream=stream)

    flush = FLUSH[name]
    sec = (time_loop_flushed if flush else time_loop)(step, steps, warmup, stream, d)
    status = kda.kda_workspace_status(ws, stream)
    if status != kda.KDA_OK:
        raise RuntimeError(f"{name}: device status {kda.kda_status_string(status)}")
    per_step = d.max(sec) / steps
    bytes_alg = prefill_bytes(th, N * H, dk, dv, q.element_size(), init is not None) + ckpt_bytes
    if variant == "gated":  # the decay logits are bf16 (2 B) where the log-decays are fp32 (4 B)
        bytes_alg -= th * dk * (4 - g.element_size())
    flops_alg = prefill_flops(th, dk, dv)
    achieved = bytes_alg / per_step / 1e9
    peak = peaks["hbm_gbs"]
    t_roof = max(bytes_alg / (peak * 1e9), flops_alg / (peaks["bf16_tflops"] * 1e12))
    traffic = None
    if with_traffic:
        prof, src = TRAFFIC_PROFILES["kda_fwd_tc_kernel"]
        fixed = N * H * dk * dv * 4 * (2 if init is not None else 1)
        traffic = scaled_traffic(prof, src, th, fixed)
    res = {"workload": spec.name + (f"_{variant}" if variant else ""), "value": job_throughput(d, th * steps, sec) / 1e6, "unit": UNIT,
           "ms_per_step": per_step * 1e3, "steps": steps, "sequences": N, "token_heads": th,
           "l2": ("flushed before every launch (256 MB write)" if flush else
                  "inputs larger than L2 (%.1f GB per step), no flush" % (bytes_alg / 1e9)),
           "pct_of_roofline": 100.0 * t_roof / per_step,
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "traffic": traffic, "bytes_per_launch": bytes_alg,
                        "kernel": "kda_fwd_tc_kernel",
                        "tensor_tflops": flops_alg / per_step / 1e12,
                        "tensor_frac_of_bf16_peak": flops_alg / per_step / 1e12 / peaks["bf16_tflops"]},
           "gpu_launches": steps * launches, **extra}
    if variant == "cp":
        res["roofline"]["kernel"] = "kda_fwd_tc_kernel state pass (segment mode) + composition + kda_fwd_tc_kernel from incoming states"
    del out, fin, ws
    return res, inp


def run_native(args, d):
    import torch

    import gated_delta_rule_121_b200 as kda
    import synth

    torch.cuda.set_device(d.local)
    dev = torch.device("cuda", d.local)
    d.init("nccl")
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid).replace("GPU-", "")

    with ClockSampler(uuid) as clk:
        main, inp = bench_prefill(args.workload, d, dev, stream, peaks, kda, synth, args.steps, args.warmup,
                                  with_traffic=args.workload == "prefill64k")
    q, v = inp["q"], inp["v"]
    B, T, H, dk = q.shape
    spec = workload_spec(args.workload)
    main["roofline"]["peak_source"] = peak_src
    line = {"metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": d.world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if q.dtype == torch.bfloat16 else "f32",
            "data": "synthetic",
            "config": {"workload": spec.name, "B": B, "T": T, "H": H, "dk": dk, "dv": v.shape[-1],
                       "sequences": main["sequences"], "chunk": CHUNK, "l2": main["l2"],
                       "parallelism": f"dp{d.world} independent replicas, no collective"},
            "pct_of_roofline": main["pct_of_roofline"], "roofline": main["roofline"],
            "gpu_launches": main["gpu_launches"], "clocks": clk.summary()}

    if not args.no_e2e:
        line["e2e"] = bench_e2e(args, d, dev, stream, inp, kda, B * T * H)
    del inp
    torch.cuda.empty_cache()
    if not args.no_decode:
        line["decode"] = bench_decode(args, d, dev, stream, peaks, kda, synth)
        line["decode_gated"] = bench_decode(args, d, dev, stream, peaks, kda, synth, gated=True)
        line["decode_spec"] = bench_spec(args, d, dev, stream, peaks, kda, synth)
    if not args.no_workloads:
        others = {}
        for key, name, steps, variant in (("mid", "mid", 50, None), ("mid_cp", "mid", 50, "cp"),
                                          ("tp4", "tp4", 10, None), ("tp4_cp", "tp4", 20, "cp"),
                                          ("varlen", "varlen", 8, None), ("stress", "stress", 50, None),
                                          ("prefill64k_model_range", "prefill64k_model_range", 5, None),
                                          ("prefill64k_ckpt512", "prefill64k", 10, "ckpt512"),
                                          ("prefill64k_gated", "prefill64k", 10, "gated")):
            if name == args.workload and variant is None:
                continue
            res, _ = bench_prefill(name, d, dev, stream, peaks, kda, synth, steps, args.warmup, variant=variant)
            others[key] = res
            torch.cuda.empty_cache()
        others["kcp8_rank"] = bench_kcp_rank(args, d, dev, stream, kda, synth, main["ms_per_step"])
        torch.cuda.empty_cache()
        line["workloads"] = others
    if d.world == 1 and d.rank == 0 and not args.no_cpu_baseline:
        import oracle
        line["cpu_baseline"] = {k: v for k, v in oracle_sample(spec, 12.0, oracle.default_threads()).items()
                                if k != "seconds"}
    if d.rank == 0:
        print(json.dumps(line), flush=True)
    d.close()


def bench_decode(args, d, dev, stream, peaks, kda, synth, gated=False):
    """One decode step per timed step over the B=512, H=96 workload; gated:
    kda_decode_step_gated on the raw prologue inputs (bf16 decay logits)."""
    import torch
    spec = synth.DECODE
    state = synth.make_decode_state(spec, dev)
    n_in = args.warmup + args.steps
    if gated:
        xs = [{n: t[:, 0].contiguous() for n, t in synth.make_spec_window(spec, s, 1, dev, prologue=True).items()}
              for s in range(n_in)]
        A_log = torch.zeros(spec.H, dtype=torch.float32, device=dev)
    else:
        xs = [synth.make_decode_step(spec, s, dev) for s in range(n_in)]
    out = torch.empty((spec.B, spec.H, spec.dv), dtype=spec.dtype, device=dev)
    it = iter(range(10 ** 9))

    def step():
        x = xs[next(it) % n_in]
        if gated:
            kda.kda_decode_step_gated(x["q"], x["k"], x["v"], x["g"], A_log, x["beta"], state, out=out,
                                      stream=stream)
        else:
            kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state, out=out, stream=stream)

    sec = time_loop(step, args.steps, args.warmup, stream, d)
    value = job_throughput(d, spec.B * spec.H * args.steps, sec) / 1e6
    per = d.max(sec) / args.steps
    nbytes = decode_bytes(spec.B, spec.H, spec.dk, spec.dv, 2)
    if gated:
        nbytes -= spec.B * spec.H * spec.dk * 2  # bf16 decay logits in place of fp32 log-decays
    ach = nbytes / per / 1e9
    prof, src = TRAFFIC_PROFILES["kda_decode_kernel"]
    traffic = None if gated else scaled_traffic(prof, src, spec.B * spec.H, 0.0)
    del xs, state
    return {"workload": spec.name + ("_gated" if gated else ""), "value": value, "unit": UNIT,
            "ms_per_step": per * 1e3, "gpu_launches": args.steps,
            "l2": "state 3.2 GB per step, far larger than L2, no flush",
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "bytes_per_launch": nbytes,
                         "kernel": "kda_decode_kernel<128,128,bf16>"}}


def bench_kcp_rank(args, d, dev, stream, kda, synth, one_gpu_ms, R=8, steps=10):
    """One rank's compute of KDA context parallelism across R ranks (KCP) for
    the 64K prefill (B=1, H=96): the rank holds 65536 / R consecutive tokens
    and runs its segment pieces (zero-start outputs and state, transformed
    queries, transition), the composition of the R gathered pieces in rank
    order and the correction of its outputs.  The all-gather of (M, S~)
    between the pieces and the composition needs R GPUs and is not timed:
    its bytes per rank are reported.  speedup_compute_only = the one-GPU
    prefill's time over this rank's."""
    import torch
    spec = synth.PRETRAIN
    T, H, dk, dv = spec.T // R, spec.H, spec.dk, spec.dv
    inp = synth.make_prefill(spec, dev, T=T)
    q, k, v, g, beta = inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"]
    out_zero = torch.empty((1, T, H, dv), dtype=torch.float32, device=dev)
    qhat = torch.empty((1, T, H, dk), dtype=torch.float32, device=dev)
    s_zero = torch.empty((R, H, dk, dv), dtype=torch.float32, device=dev)  # this rank's piece + the gathered ones
    trans = torch.empty((R, H, dk, dk), dtype=torch.float32, device=dev)
    state_in = torch.empty_like(s_zero)
    final = torch.empty((1, H, dk, dv), dtype=torch.float32, device=dev)
    out = torch.empty((1, T, H, dv), dtype=spec.dtype, device=dev)
    ws = kda.alloc_workspace(1, T, H, dk, dv, spec.dtype, dev)
    lib, ptr, sp = kda.lib(), kda._ptr, kda._stream_ptr(stream)
    rank = R // 2
    # the other ranks' pieces stand in as copies of this one (the composition's
    # cost does not depend on the values)
    code = lib.kda_segment_fwd(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(out_zero), ptr(s_zero[0]),
                               ptr(qhat), ptr(trans[0]), 1, T, H, dk, dv, None, sp, kda._DT[q.dtype], ptr(ws),
                               ws.numel())
    kda._check(code, "kda_segment_fwd")
    torch.cuda.synchronize()
    s_zero[1:].copy_(s_zero[0].expand(R - 1, -1, -1, -1))
    trans[1:].copy_(trans[0].expand(R - 1, -1, -1, -1))
    s_mine, t_mine, s_in_mine = s_zero[rank], trans[rank], state_in[rank]

    def step():
        kda._check(lib.kda_segment_fwd(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(out_zero), ptr(s_mine),
                                       ptr(qhat), ptr(t_mine), 1, T, H, dk, dv, None, sp, kda._DT[q.dtype],
                                       ptr(ws), ws.numel()), "kda_segment_fwd")
        kda._check(lib.kda_state_compose(ptr(trans), ptr(s_zero), None, ptr(state_in), ptr(final), R, 1, H, dk, dv,
                                         1, sp), "kda_state_compose")
        kda._check(lib.kda_output_correct(ptr(out_zero), ptr(qhat), ptr(s_in_mine), ptr(out), 1, T, H, dk, dv, None,
                                          sp, kda._DT[out.dtype]), "kda_output_correct")

    sec = time_loop(step, steps, args.warmup, stream, d)
    ms = d.max(sec) / steps * 1e3
    gather_bytes = H * (dk * dk + dk * dv) * 4
    res = {"workload": f"kcp_rank_of_{R}_prefill_bf16_B1_H{H}_T{spec.T}_d{dk}", "tokens_per_rank": T,
           "value": job_throughput(d, T * H * steps, sec) / 1e6, "unit": UNIT, "ms_per_step": ms,
           "gpu_launches": 3 * steps, "speedup_compute_only": one_gpu_ms / ms,
           "allgather": {"bytes_sent_per_rank": gather_bytes, "bytes_received_per_rank": (R - 1) * gather_bytes,
                         "timed": False, "why": "needs R GPUs; one here"}}
    del inp, q, k, v, g, beta, out_zero, qhat, s_zero, trans, state_in, final, out, ws
    return res


def bench_spec(args, d, dev, stream, peaks, kda, synth, W=4, sweep=(1, 2, 4, 8)):
    """Speculative verification with state replay at B=512, H=96: every step
    replays the accepted drafts of the previous window (accept counts drawn
    uniformly in 0..W-1, seeded), runs the bonus token and W-1 new drafts, and
    writes the state once.  value = new-window tokens x heads per second;
    the roofline counts the state read and write plus the token bytes read.
    Also the step time for windows of 1, 2, 4 and 8 tokens (the verification
    cost against the number of tokens it covers)."""
    import numpy as np
    import torch
    spec = synth.DECODE
    B, H, dk, dv = spec.B, spec.H, spec.dk, spec.dv
    rng = np.random.default_rng(9)
    res = {"workload": f"spec_decode_bf16_B{B}_H{H}_d128_W{W}"}
    times = {}
    for w in sorted(set(sweep) | {W}):
        state = synth.make_decode_state(spec, dev)
        n_in = args.warmup + args.steps + 1
        wins = [synth.make_spec_window(spec, s, w, dev) for s in range(n_in)]
        accs = [torch.tensor(rng.integers(0, w, B), dtype=torch.int32, device=dev) for _ in range(n_in)]
        out = torch.empty((B, w, H, dv), dtype=spec.dtype, device=dev)
        it = iter(range(10 ** 9))

        def step():
            i = next(it) % (n_in - 1)
            kda.kda_decode_spec(wins[i], accs[i], wins[i + 1], state, out=out, stream=stream)

        sec = time_loop(step, args.steps, args.warmup, stream, d)
        times[w] = d.max(sec) / args.steps
        if w == W:
            mean_acc = float(torch.stack(accs).float().mean())
            nbytes = B * H * (2 * dk * dv * 4 + (w + mean_acc) * (2 * (2 * dk + dv) + 4 * dk + 4) + w * 2 * dv)
            ach = nbytes / times[w] / 1e9
            prof, src = TRAFFIC_PROFILES["kda_spec_kernel"]
            traffic = scaled_traffic(prof, src, B * H, 0.0)
            res.update(value=job_throughput(d, B * H * w * args.steps, sec) / 1e6, unit=UNIT,
                       ms_per_step=times[w] * 1e3, mean_accepted=mean_acc, gpu_launches=args.steps,
                       roofline={"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                 "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "bytes_per_launch": nbytes,
                                 "kernel": "kda_spec_kernel<128,128,bf16>"})
        del wins, accs, state, out
        torch.cuda.empty_cache()
    res["ms_per_step_by_window"] = {str(w): t * 1e3 for w, t in sorted(times.items())}
    return res


def bench_e2e(args, d, dev, stream, inp, kda, th):
    """Same metric through the C entry point kda_fwd_host from pinned host
    buffers: every step copies the inputs host->device and the output and
    final state back, all enqueued by that one call."""
    import torch
    host = {n: (t.cpu().pin_memory() if t is not None else None) for n, t in inp.items()}
    bufs = {}
    steps = max(1, min(args.steps, 5))

    def step():
        kda.kda_fwd_host(host["q"], host["k"], host["v"], host["g"], host["beta"], host["init_state"],
                         host["cu_seqlens"], device=dev, stream=stream, dev_buffers=bufs)

    step()  # allocates the device buffers outside the timed region
    sec = time_loop(step, steps, args.warmup, stream, d)
    h2d = sum(t.numel() * t.element_size() for n, t in host.items() if t is not None)
    d2h = bufs["out_h"].numel() * bufs["out_h"].element_size() + bufs["fin_h"].numel() * 4
    value = job_throughput(d, th * steps, sec) / 1e6
    del bufs, host
    return {"value": value, "unit": UNIT, "h2d_bytes_per_step": h2d, "entry_point": "kda_fwd_host",
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": d.max(sec) / steps * 1e3}


# Small cases for ncu counter captures (a few GB on the device at most,
# inputs larger than L2); the traffic files under profiles/ name the case.
CAPTURES = {
    "prefill_h96_t4096": "B=1 H=96 T=4096 d=128 bf16 prefill (the 64K workload's heads, 1/16 of its tokens)",
    "mid": "B=2 H=16 T=4096 d=128 bf16 prefill with initial states",
    "decode_b64_h96": "B=64 H=96 d=128 bf16 decode step (1/8 of the decode workload's sequences)",
    "spec_b64_h96_w4": "B=64 H=96 d=128 bf16 speculative verification, windows of 4, accepted drafts 0..3",
}


def run_capture(args):
    """A few launches of one small case, nothing else: the command ncu wraps."""
    import torch

    import gated_delta_rule_121_b200 as kda
    import synth
    dev = torch.device("cuda")
    n = max(1, args.steps)
    if args.capture == "spec_b64_h96_w4":
        import numpy as np
        spec, B, W = synth.DECODE, 64, 4
        state = synth.make_decode_state(spec, dev, B=B)
        wins = [synth.make_spec_window(spec, s, W, dev, B=B) for s in range(n + 1)]
        acc = torch.tensor(np.random.default_rng(9).integers(0, W, B), dtype=torch.int32, device=dev)
        for i in range(n):
            kda.kda_decode_spec(wins[i], acc, wins[i + 1], state)
    elif args.capture == "decode_b64_h96":
        spec = synth.DECODE
        state = synth.make_decode_state(spec, dev, B=64)
        x = synth.make_decode_step(spec, 0, dev, B=64)
        for _ in range(n):
            kda.kda_decode_step(x["q"], x["k"], x["v"], x["g"], x["beta"], state)
    else:
        spec = synth.PRETRAIN if args.capture == "prefill_h96_t4096" else synth.MID
        inp = synth.make_prefill(spec, dev, T=4096)
        for _ in range(n):
            kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], inp["cu_seqlens"])
    torch.cuda.synchronize()
    print(json.dumps({"capture": args.capture, "what": CAPTURES[args.capture], "launches": n}), flush=True)


# Phase boundaries recorded by the tensor-core kernel's test hook (chain 0):
# (name, from event, to event) per group; see include/kda_testing.h.
PHASES = {
    "front": [("decay_prefix", 0, 1), ("stage_wait", 1, 2), ("scale_q_k_v", 2, 3), ("buffer_wait", 3, 4),
              ("kh", 4, 5), ("g1_issue", 5, 6), ("g1_wait", 6, 7), ("p_a_tiles", 7, 26)],
    "back": [("front_wait", 16, 17), ("diag_inverses", 17, 18), ("y_f", 18, 19), ("x", 19, 20),
             ("t10_tprime", 20, 21), ("g2_g3_issue", 21, 22), ("g2_g3_wait", 22, 23), ("w_tile", 23, 25)],
    "scan": [("d2_wait", 8, 9), ("s_pass", 9, 10), ("d1a", 10, 27), ("back_wait", 27, 24), ("d1b", 24, 11),
             ("tma", 11, 28), ("d1_wait", 28, 13), ("delta", 13, 14), ("d2_issue", 14, 15), ("output", 15, 12)],
}


def run_phases(args):
    """Per-phase SM cycles of chain 0 (chunks 8..59), from the test hook."""
    import numpy as np
    import torch

    import gated_delta_rule_121_b200 as kda
    import synth
    spec = workload_spec(args.workload)
    inp = synth.make_prefill(spec, torch.device("cuda"))
    dbg = torch.zeros(kda.lib().kda_testing_debug_floats(), dtype=torch.float32, device="cuda")
    for _ in range(args.warmup):
        kda.kda_fwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], inp["cu_seqlens"],
                    _debug=dbg)
    torch.cuda.synchronize()
    t = dbg[61568:].cpu().numpy().view(np.int64).reshape(64, 32)
    cu = inp["cu_seqlens"]
    n0 = int(cu[1] - cu[0]) if cu is not None else inp["q"].shape[1]
    hi = min(60, (n0 + CHUNK - 1) // CHUNK)  # chunks of chain 0 with timestamps, skipping the ramp
    lo = min(8, hi // 2)
    res = {"workload": spec.name, "chunks": [lo, hi], "unit": "SM cycles per chunk (chain 0)"}
    for grp, ph in PHASES.items():
        res[grp] = {n: float(np.mean(t[lo:hi, b] - t[lo:hi, a])) for n, a, b in ph}
    res["period"] = float(np.mean(np.diff(t[lo:hi, 0])))
    print(json.dumps(res), flush=True)


def run_chains(args):
    """Prefill over H independent heads (one chain each, B=1) for each H in
    --chains: kernel time per 64-token chunk (median of --steps launches) and
    chain 0's own chunk period in SM cycles (test hook).  The two diverge when
    some chains run slower than chain 0."""
    import numpy as np
    import torch

    import gated_delta_rule_121_b200 as kda
    import synth
    T = args.chain_tokens
    for H in (int(h) for h in args.chains.split(",")):
        spec = synth.PrefillSpec(f"chains_H{H}_T{T}", 1, T, H, 128, 128, torch.bfloat16, 2)
        inp = synth.make_prefill(spec, torch.device("cuda"))
        call = (inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"], inp["init_state"], inp["cu_seqlens"])
        out = torch.empty_like(inp["q"])
        fin = torch.empty(1, H, 128, 128, device="cuda")
        ws = kda.alloc_workspace(1, T, H, 128, 128)
        for _ in range(args.warmup):
            kda.kda_fwd(*call, out=out, final_state=fin, workspace=ws)
        torch.cuda.synchronize()
        ms = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            kda.kda_fwd(*call, out=out, final_state=fin, workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        med = float(np.median(ms))
        res = {"chains": H, "tokens": T, "ms": med, "us_per_chunk": med * 1e3 / (T // CHUNK)}
        if not args.no_period:
            dbg = torch.zeros(kda.lib().kda_testing_debug_floats(), dtype=torch.float32, device="cuda")
            kda.kda_fwd(*call, out=out, final_state=fin, workspace=ws, _debug=dbg)
            torch.cuda.synchronize()
            t = dbg[61568:].cpu().numpy().view(np.int64).reshape(64, 32)
            hi = min(60, T // CHUNK)
            res["chain0_period_cycles"] = float(np.mean(np.diff(t[min(8, hi // 2):hi, 0])))
        print(json.dumps(res), flush=True)
        del inp, out, fin, ws
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=["prefill64k", "mid", "varlen", "stress", "tp4", "prefill64k_model_range"],
                    default="prefill64k")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other workload objects (mid, tp4, varlen, stress, model range, checkpoints, gated, KCP rank)")
    ap.add_argument("--capture", choices=sorted(CAPTURES), default=None,
                    help="run --steps launches of a small case (for ncu), nothing else")
    ap.add_argument("--phases", action="store_true",
                    help="print per-phase cycles of the tensor-core kernel (test hook) instead of timing")
    ap.add_argument("--chains", default=None,
                    help="comma-separated head counts: time B=1 prefills with that many chains instead")
    ap.add_argument("--chain-tokens", type=int, default=16384)
    ap.add_argument("--no-period", action="store_true", help="with --chains: skip the test-hook launch")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    d = Dist()
    if args.capture:
        run_capture(args)
    elif args.phases:
        run_phases(args)
    elif args.chains:
        run_chains(args)
    elif args.impl == "reference":
        run_reference(args, d)
    else:
        run_native(args, d)


if __name__ == "__main__":
    main()
