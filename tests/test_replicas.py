"""The replicas plumbing of bench.py (one process per GPU, no data exchange) on CPU:
two gloo ranks agree on the max over ranks, the whole-job rate counts every rank's
units, and only rank 0 prints; the reference arm's other ranks exit without work."""
import io
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch
    import bench
    rep = bench.Replicas(world, rank, backend="gloo", device=torch.device("cpu"), timeout_s=60)
    rep.barrier()
    ms = rep.max_over_ranks(1.0 + rank)          # rank r "took" 1 + r ms
    rate = rep.whole_job_rate(64, ms)
    buf = io.StringIO()
    with redirect_stdout(buf):
        rep.emit({"rank": rank, "value": rate})
    rep.barrier()
    rep.close()
    q.put((rank, ms, rate, buf.getvalue()))


def test_two_gloo_ranks_max_time_whole_job_rate_rank0_prints():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, rate0, out0), (r1, ms1, rate1, out1) = res
    assert ms0 == ms1 == 2.0                       # the slowest rank's time on every rank
    assert rate0 == rate1 == pytest.approx(2 * 64 / 2e-3)
    assert '"rank": 0' in out0 and out1 == ""


def test_reference_arm_other_ranks_exit_without_work():
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        steps, warmup = 2, 3

    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.bench_reference(Args(), 2, 1) == 0
    assert buf.getvalue() == ""
