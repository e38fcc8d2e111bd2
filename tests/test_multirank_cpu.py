"""The multi-GPU host path of bench.py (replicas: a barrier and the max over ranks of the
timings, no data-path collective) on two CPU ranks over gloo, and the reference arm's rank
behaviour under torchrun (only rank 0 runs and prints)."""
import contextlib
import io
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        ws, r, local = bench.dist_setup(None, backend="gloo")
        bench.barrier(ws)
        ms = [3.0, 5.0][rank]                       # rank 1 is the slow one
        m = bench.max_over_ranks(ws, ms)
        bench.barrier(ws)
        q.put((r, ws, local, m, bench.job_value(ws, 1e12, 10, m)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 for g in got)
    assert [g[2] for g in got] == [0, 1]
    assert all(g[3] == 5.0 for g in got)             # both ranks see the max
    # whole-job value: 2 ranks x 10 steps x 1 TFLOP in 5 ms
    assert all(abs(g[4] - 2 * 10 * 1.0 / 5e-3) < 1e-9 for g in got)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(1, 7.5) == 7.5
    assert bench.job_value(1, 2e12, 4, 8.0) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    out = io.StringIO()
    with contextlib.redirect_stdout(out):
        assert bench.run_reference(bench.argparse.Namespace(steps=3, warmup=3)) is None
    assert out.getvalue() == ""
