"""The benchmark's multi-rank host logic on CPU: two gloo ranks (the replicas
a torchrun launch of bench.py starts, one per GPU) meet at the barrier, agree
on the slowest rank's time, and report the whole job's throughput; the
reference arm runs on rank 0 alone."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench._sync_barrier(True)
        slowest = bench._max_over_ranks(1.0 + rank, True)      # rank r "took" 1 + r seconds
        rate = bench.aggregate_rate(world, 1000, 5, slowest)
        out[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_rank_and_sum_the_work():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    slowest, rate = res[0]
    assert slowest == 2.0
    assert rate == pytest.approx(2 * 1000 * 5 / 2.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    calls = []
    monkeypatch.setattr(bench, "run_reference", lambda *a: calls.append(a))
    for rank in (1, 0):
        monkeypatch.setenv("WORLD_SIZE", "2")
        monkeypatch.setenv("RANK", str(rank))
        monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2"])
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.main()
        assert buf.getvalue() == ""
    assert len(calls) == 1 and calls[0][2] == 0   # (args, cfg, rank, world): rank 0
