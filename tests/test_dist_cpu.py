"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank processes its own batch (weak scaling, no collective on the data
path); the only collective is the max over ranks of the timed step, and the
whole-job value is all ranks' units over that max."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        seconds = [0.010, 0.013][rank]            # rank 1 is the slow one
        smax = bench.max_over_ranks(seconds, "cpu")
        value = bench.aggregate(3.0e12, w, smax)
        out.put((rank, smax, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling_value():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(2))
    for rank, smax, value in got:
        assert smax == pytest.approx(0.013)
        assert value == pytest.approx(2 * 3.0e12 / 0.013)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3"])
    assert capsys.readouterr().out == ""
