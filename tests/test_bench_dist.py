"""The multi-GPU path of bench.py, run as world_size-2 gloo ranks on CPU:
the timing barrier, the max-over-ranks time and the whole-job throughput
(all ranks' units over the slowest rank's time), and the reference arm's
rule that only rank 0 runs the oracle."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo", timeout_s=60)
    try:
        d.barrier()
        secs = [2.0, 3.0][rank]        # this rank's own device time
        units = [100.0, 100.0][rank]   # weak scaling: the same work per rank
        res = dict(rank=rank, max=d.max(secs), sum=d.sum(units),
                   rate=bench.job_throughput(d, units, secs))
        # the reference arm returns at once on every rank but 0, without work
        if rank == 1:
            class A:
                workload, steps, warmup, gpus = "prefill64k", 1, 3, world
            res["ref_rank1"] = bench.run_reference(A, d)
        d.barrier()
        q.put(res)
    finally:
        d.close()


def test_two_rank_aggregation_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted([q.get(timeout=120) for _ in ps], key=lambda r: r["rank"])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in res:
        assert r["max"] == pytest.approx(3.0)    # the slowest rank's time
        assert r["sum"] == pytest.approx(200.0)  # all ranks' units
        assert r["rate"] == pytest.approx(200.0 / 3.0)
    assert res[1]["ref_rank1"] is None


def test_single_process_aggregation_is_local():
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.world, d.rank = 1, 0
    d.init("gloo")
    assert d.pg is None
    assert bench.job_throughput(d, 50.0, 2.0) == pytest.approx(25.0)
