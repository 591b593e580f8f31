"""Host-side logic of bench.py for several ranks, on CPU with gloo
(world size 2): the slowest rank's time is reported, throughput aggregates
over ranks, and only rank 0 of the reference arm prints."""
import json
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 1.0 + rank  # rank 1 is the slow one
        slowest = bench.max_over_ranks(torch, mine, dist, device="cpu")
        rate = bench.whole_job_rate(10.0, 4, world, slowest)
        results[rank] = (slowest, rate)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_rate():
    world = 2
    port = _free_port()
    with mp.Manager() as manager:
        results = manager.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        got = dict(results)
    for rank in range(world):
        slowest, rate = got[rank]
        assert slowest == 2.0  # every rank sees the slowest rank's time
        assert rate == pytest.approx(10.0 * 4 * world / 2.0)


def test_reference_arm_prints_only_on_rank_zero(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setattr(sys, "argv", ["bench.py", "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"])
    assert bench.main() == 0
    assert capsys.readouterr().out == ""


def test_single_process_rate():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(torch, 0.5, None, device="cpu") == 0.5
    assert bench.whole_job_rate(2.0, 3, 1, 0.5) == 12.0
