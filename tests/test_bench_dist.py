"""The N > 1 path of bench.py, on CPU: two gloo ranks on 127.0.0.1.

Under torchrun every GPU runs its own copy of the step (replicas, weak
scaling); the step time is the slowest rank's, the reported value counts the
work of all ranks, and only rank 0 prints.  The reference arm runs the oracle
on rank 0 alone; the other ranks exit without work.  These are the pieces of
that path that need no GPU, run here through the same helpers bench.py uses.
"""
import datetime
import os
import socket
import sys

import pytest

from conftest import ROOT


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, root, out):
    sys.path.insert(0, root)
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = (12.5, 20.0)[rank]           # this rank's own step time
        slowest = bench.max_over_ranks(local_ms, world)
        value = bench.whole_job_tflops(world, 1.0e12, slowest)
        dist.barrier()
        out.put((rank, slowest, value, bench.reports(rank)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, ROOT, out)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(out.get(timeout=180) for _ in range(2))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    (r0, t0, v0, p0), (r1, t1, v1, p1) = got
    assert (r0, r1) == (0, 1)
    assert t0 == t1 == 20.0                      # max over ranks, seen by both
    assert v0 == v1 == pytest.approx(2 * 1.0e12 / 0.020 / 1e12)
    assert (p0, p1) == (True, False)             # one JSON line, from rank 0


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1) == 7.0
    assert bench.whole_job_tflops(1, 3.0e12, 1000.0) == pytest.approx(3.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    # returns before it reads its arguments or touches the oracle
    assert bench.run_reference(None, None) == 0
