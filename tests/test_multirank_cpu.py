"""The multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

Each rank reports its own timing; the job's throughput must be all ranks'
work over the slowest rank's time (weak scaling: every rank runs the same
per-rank step), and the reference arm must run on rank 0 only.  Failures
are made on the host: a rank that raises after joining, and a rank that
never joins; the surviving rank must end with an error, not hang.
"""
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


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    d = bench.Dist()
    d.init("gloo")
    d.barrier()
    # rank r pretends its timed region took (r + 1) * 100 ms for 7 units of work
    rate, ms = d.aggregate(7.0, (rank + 1) * 100.0)
    ref_rank_runs = bench.Dist().rank == 0
    d.barrier()
    q.put((rank, rate, ms, ref_rank_runs))
    d.close()


def test_two_gloo_ranks_aggregate_weak_scaling():
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
    for rank, rate, ms, ref_runs in res:
        assert ms == pytest.approx(200.0)              # max over ranks
        assert rate == pytest.approx(2 * 7.0 / 0.2)    # both ranks' units / slowest time
        assert ref_runs == (rank == 0)


def test_reference_arm_skips_nonzero_ranks(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class A:
        ref_rows = 1
        warmup = 0
        steps = 1
        gpus = 2
    assert bench.run_reference(A(), bench.Dist()) is None


def _failing_worker(rank, world, port, q, mode):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), HYB_PG_TIMEOUT_S="5")
    sys.path.insert(0, ROOT)
    import time
    import bench
    if rank == 1 and mode == "never_joins":
        q.put((rank, "absent", 0.0))
        return
    d = bench.Dist()
    t0 = time.monotonic()
    try:
        d.init("gloo")
        if rank == 1:
            raise RuntimeError("rank 1 fails between steps")
        d.barrier()
        d.max(1.0)
        q.put((rank, "completed", time.monotonic() - t0))
    except RuntimeError as e:
        q.put((rank, "error" if rank == 0 else "raised", time.monotonic() - t0))
        if rank == 1:   # leave without tearing the group down, as a crashed rank would
            q.close()
            q.join_thread()
            os._exit(3)


@pytest.mark.parametrize("mode", ["raises_after_join", "never_joins"])
def test_surviving_rank_errors_instead_of_hanging(mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_worker, args=(r, 2, port, q, mode)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (status, t)) for r, status, t in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
    status0, t0 = res[0]
    assert status0 == "error", res
    assert t0 < 60.0, res
