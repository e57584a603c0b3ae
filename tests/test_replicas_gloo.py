"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The layer has no exchange step, so `--gpus N` runs N independent replicas:
the only collectives are a barrier and a max of the per-rank times, and the
whole-job throughput is the units all ranks processed over the slowest
rank's time.  These tests run that host logic in two processes over gloo.
"""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica(rank, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE="2",
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    world, r, local = bench.dist_setup()
    d = bench.Dist(world, r, local, backend="gloo", timeout_s=60)
    try:
        d.barrier()
        # rank 1 is the slower replica: 15 ms for the same 100 units
        units_per_s, ms_max = bench.aggregate(100.0, 10.0 + 5.0 * r, d)
        q.put((r, units_per_s, ms_max, d.max(float(r))))
    finally:
        d.close()


def test_two_replicas_report_the_slowest_rank_and_the_summed_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_replica, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert [p.exitcode for p in procs] == [0, 0]
    for rank, units_per_s, ms_max, mx in got:
        assert ms_max == 15.0            # max over ranks, seen by every rank
        assert units_per_s == pytest.approx(2 * 100.0 / 0.015)
        assert mx == 1.0


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), {"gpus": 2, "steps": 1, "warmup": 0, "cpu_rows": 1})()
    assert bench.reference_arm(args) is None
    assert capsys.readouterr().out == ""
