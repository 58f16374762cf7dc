"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

The layer shards by replicas only (independent tokens; each rank runs the
whole workload on its own GPU, no data-path collective), so what multi-GPU
adds is the timing plumbing: a barrier on both sides of the timed region,
the slowest rank's time (max over ranks), and the whole-job rate computed
from it.  These tests run that plumbing with world_size 2 and check the
reference arm's rank handling (rank 0 alone runs it)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _env(rank: int, world: int, port: int):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))


def _timing_worker(rank: int, world: int, port: int, q):
    try:
        import sys
        sys.path.insert(0, ROOT)
        _env(rank, world, port)
        import bench
        d = bench.Dist(world, backend="gloo")
        assert (d.world, d.rank) == (world, rank)
        d.barrier()
        t = d.max(1.0 + 0.5 * rank)              # rank r "took" 1 + r/2 seconds
        d.barrier()
        rate = bench.whole_job_rate(d.world, 10, 100.0, t)
        d.close()
        q.put((rank, t, rate, None))
    except Exception as e:                       # report instead of hanging the parent
        q.put((rank, None, None, repr(e)))


def _reference_worker(rank: int, world: int, port: int, q):
    try:
        import contextlib
        import io
        import sys
        sys.path.insert(0, ROOT)
        _env(rank, world, port)
        import bench
        if rank == 0:
            q.put((rank, "skip", None))          # rank 0 would run the oracle step
            return
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            args = bench.argparse.Namespace(gpus=world, steps=1, warmup=1)
            rc = bench.run_reference(args)
        q.put((rank, rc, buf.getvalue()))
    except Exception as e:
        q.put((rank, "error", repr(e)))


def _run(target, world=2, timeout=120):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = [q.get(timeout=timeout) for _ in range(world)]
    for p in procs:
        p.join(timeout=timeout)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not exit")
    return sorted(out, key=lambda r: r[0])


def test_replica_timing_is_the_max_over_ranks():
    res = _run(_timing_worker)
    for rank, t, rate, err in res:
        assert err is None, f"rank {rank}: {err}"
        assert t == 1.5                          # every rank sees the slowest rank's time
        assert rate == pytest.approx(2 * 10 * 100.0 / 1.5)


def test_whole_job_rate_is_weak_scaling():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_rate(1, 20, 17107232.0, 0.001)
    eight = bench.whole_job_rate(8, 20, 17107232.0, 0.001)
    assert eight == pytest.approx(8 * one)       # same per-rank work and time


def test_reference_arm_runs_on_rank_zero_only():
    res = _run(_reference_worker)
    assert res[0][1] == "skip"
    rank, rc, printed = res[1]
    assert rc == 0 and printed == "", (rc, printed)
