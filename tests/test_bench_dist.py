"""Multi-rank plumbing of bench.py on CPU (gloo, world size 2): the timing
reduction takes the slowest rank, the whole-job value counts every rank's
units, and the reference arm does its work on rank 0 only."""
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    bench.init_dist(world, "gloo")
    ms = [3.0, 5.0][rank]
    slowest = bench.max_over_ranks(ms, world)
    bench.barrier(world)
    value = bench.aggregate_value(1e12, world, slowest * 1e-3)
    import torch.distributed as dist
    dist.destroy_process_group()
    q.put((rank, slowest, value))


def test_max_over_ranks_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value in res:
        assert slowest == 5.0                      # max over ranks, on every rank
        assert value == pytest.approx(2e12 / 5e-3)  # both ranks' units / slowest time


def test_reference_arm_other_ranks_do_no_work(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    called = []
    monkeypatch.setattr(bench, "_oracle_sample", lambda *a, **k: called.append(1))
    bench.run_reference(bench.parse_args(["--impl", "reference", "--steps", "1", "--warmup", "0"]))
    assert not called
    assert capsys.readouterr().out == ""
