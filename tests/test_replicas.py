"""Replica timing logic of bench.py on two gloo ranks (CPU).

The method has no exchange step, so N GPUs run N independent replicas; the
only cross-rank work is the barrier around the timed region and the maximum
of the per-rank times.  These tests run that logic as two processes on the
gloo backend.
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
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench._barrier(world)
        # Each rank reports its own time; every rank must see the maximum.
        got = bench._max_over_ranks(1.5 + rank, world)
        bench._barrier(world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=5) for _ in range(world))
    assert res == {0: 2.5, 1: 2.5}


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench

    assert bench._max_over_ranks(3.25, 1) == 3.25
    bench._barrier(1)  # no-op without a process group


def test_reference_arm_other_ranks_exit_without_work(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("RANK", "1")

    class A:
        steps, warmup, gpus = 1, 3, 2

    def boom(*a, **k):
        raise AssertionError("rank 1 must not run the oracle")

    monkeypatch.setattr(bench, "cpu_baseline", boom)
    assert bench.run_reference(A()) == 0


@pytest.mark.parametrize("warmup", [0, 2])
def test_bench_rejects_short_warmup(warmup, monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setattr(sys, "argv", ["bench.py", "--warmup", str(warmup)])
    with pytest.raises(SystemExit):
        bench.main()
