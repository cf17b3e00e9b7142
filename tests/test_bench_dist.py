"""The benchmark's multi-process plumbing on CPU (gloo, world size 2): rank
bookkeeping, the barrier-bracketed timed region and the max over ranks that the
reported time is. The GPU work itself is replaced by a fake step here."""
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


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist(world, backend="gloo")
    try:
        calls = []

        def run():
            calls.append(rank)
            return 0.25 * (rank + 1)  # rank 1 is the slow one

        secs = bench.timed_region(d, run, lambda: None)
        q.put((rank, secs, d.rank, d.world, len(calls)))
    finally:
        d.close()


def test_timed_region_reports_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    for rank, secs, drank, dworld, ncalls in res:
        assert secs == pytest.approx(0.5)   # both ranks see the slowest rank's time
        assert drank == rank and dworld == 2 and ncalls == 1


def test_world_size_must_match_gpus(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    with pytest.raises(SystemExit):
        bench.Dist(1)


def _ref_rank_main(rank, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE="2")
    sys.path.insert(0, ROOT)
    import bench

    class A:
        steps, warmup = 1, 3
    q.put((rank, bench.run_reference(A, rank, 2) is None))


def test_reference_arm_runs_on_rank_zero_only():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_ref_rank_main, args=(1, q))
    p.start()
    rank, is_none = q.get(timeout=60)
    p.join(timeout=60)
    assert p.exitcode == 0 and rank == 1 and is_none
