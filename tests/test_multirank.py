"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2):
per-rank seeds, max-over-ranks timing and the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        own = [10.0 + rank, 5.0 - rank, 1.0 * rank]
        got = bench.max_over_ranks(own, world)
        seed = bench.rank_seed(1005, rank)
        seeds = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(seeds, torch.tensor([seed]))
        out[rank] = (got, [int(x) for x in seeds])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timings_and_distinct_seeds():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        got, seeds = res[r]
        assert got == [11.0, 5.0, 1.0]
        assert seeds == [1005, 1006]


def test_whole_job_throughput_scales_with_ranks():
    one = bench.whole_job_tflops(51.9e12, 5, 1, 500.0)
    two = bench.whole_job_tflops(51.9e12, 5, 2, 500.0)
    assert one == pytest.approx(519.0) and two == pytest.approx(2 * one)
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]
