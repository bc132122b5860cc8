"""The replica bookkeeping of bench.py under two processes (gloo on CPU):
every rank's time is reduced to the slowest one, the whole-job rate counts
every rank's tokens over that time, and the reference arm runs on rank 0
only (the other ranks return without work)."""
import importlib.util
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_ranks", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _load_bench()
        ms = b.max_over_ranks(1.0 + 2.0 * rank, world)  # rank 0: 1 ms, rank 1: 3 ms
        q.put((rank, ms, b.job_rate(world, 10, 4, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, rate in got:
        assert ms == 3.0  # the slowest rank's time on every rank
        assert rate == pytest.approx(2 * 10 * 4 / 3e-3)


def test_single_rank_is_unchanged():
    b = _load_bench()
    assert b.max_over_ranks(1.25, 1) == 1.25
    assert b.job_rate(1, 30, 4096, 1.25 * 30) == pytest.approx(30 * 4096 / (1.25 * 30e-3))


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    b = _load_bench()
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
    out = io.StringIO()
    with redirect_stdout(out):
        b.main()
    assert out.getvalue() == ""
