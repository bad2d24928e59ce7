"""The multi-rank host logic (one process per GPU, weak scaling) on CPU with
gloo, world size 2: max-over-ranks timing, the job's aggregate throughput and
per-rank independent problems."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from rwkv_wkv_recurrence_b200.dist_timing import max_over_ranks, rank_seed, weak_scaling_throughput


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import wkv_inputs as wi

        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        m = max_over_ranks(local_ms)
        # each rank's problem: same shapes, different draws
        p = wi.wkv4_problem(2, 8, 32, rank_seed(7, rank), outliers=True, with_gy=True)
        gathered = [torch.zeros_like(p["k"]) for _ in range(world)]
        dist.all_gather(gathered, p["k"].contiguous())
        out[rank] = (m, weak_scaling_throughput(1000.0, world, m), bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        m, thr, same = out[r]
        assert m == 15.0, "every rank sees the slowest rank's time"
        assert thr == pytest.approx(2 * 1000.0 / 15e-3)
        assert not same, "ranks must draw independent problems"


def test_single_process_without_group():
    assert max_over_ranks(3.5) == 3.5
    assert weak_scaling_throughput(100.0, 1, 2.0) == pytest.approx(50000.0)


def test_seeds_and_validation():
    assert rank_seed(5, 0) == 5 and rank_seed(5, 3) == 3005
    with pytest.raises(ValueError):
        rank_seed(5, -1)
    with pytest.raises(ValueError):
        weak_scaling_throughput(1.0, 0, 1.0)
    with pytest.raises(ValueError):
        weak_scaling_throughput(1.0, 1, 0.0)
