"""The N > 1 host path of bench.py, as two gloo ranks on the CPU.

Under torchrun the layer runs as independent replicas (one process per GPU, no data-path
collective).  What the ranks share is host logic: the barrier around the timed region,
the max over ranks of the device times, the whole-job throughput from it, and the
reference arm, which rank 0 alone runs and prints.  These run here without a GPU.
"""
from __future__ import annotations

import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, ws: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench.barrier(ws)
        # each rank's own device time; the job ends with the slowest
        t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)
        value = bench.job_tflops(ws, 1e12, 4, t)
        # the reference arm: every rank but 0 returns at once and prints nothing
        out = io.StringIO()
        if rank != 0:
            args = type("A", (), {"steps": 1, "warmup": 0})()
            with contextlib.redirect_stdout(out):
                ret = bench.run_reference(args)
            ref = (ret, out.getvalue())
        else:
            ref = None
        bench.barrier(ws)
        q.put((rank, t, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_value():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(ws):
            rank, t, value, ref = q.get(timeout=120)
            results[rank] = (t, value, ref)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
                p.join()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    # both ranks see the slowest rank's time (15 ms), and the job's value counts both
    # ranks' work: 2 ranks x 4 steps x 1 TFLOP in 15 ms
    for rank in range(ws):
        t, value, _ = results[rank]
        assert t == pytest.approx(15.0)
        assert value == pytest.approx(2 * 4 * 1.0 / 15e-3)
    ret, printed = results[1][2]
    assert ret is None and printed == ""


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.barrier(1)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tflops(1, 2e12, 10, 20.0) == pytest.approx(1000.0)
