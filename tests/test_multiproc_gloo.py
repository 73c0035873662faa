"""The multi-rank path of bench.py on CPU: world size 2 over gloo.

Each rank of `bench.py --gpus N` runs an independent replica of the workload
(the path has no exchange step); the job's time is the slowest rank's, taken
with an all-reduce MAX, and the whole-job value divides it over every rank's
units.  These tests run that plumbing with two gloo ranks on 127.0.0.1."""

import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        bench._barrier(world)
        local_ms = [12.0, 20.0][rank]              # rank 1 is the slow one
        mx = bench._max_over_ranks(local_ms, world)
        per_unit = bench.whole_job_us_per_unit(local_ms, 10, world)
        bench._barrier(world)
        q.put((rank, mx, per_unit))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    for rank, mx, per_unit in got:
        assert mx == 20.0                                  # max over ranks
        assert per_unit == pytest.approx(20.0e3 / 20)      # 20 ms over 2 x 10 units


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench._max_over_ranks(3.5, 1) == 3.5
    assert bench.whole_job_us_per_unit(3.0, 6, 1) == pytest.approx(500.0)


def test_reference_arm_on_other_ranks_exits_without_work(monkeypatch, capsys):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"]) == 0
    assert capsys.readouterr().out == ""
