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
        h0, nh = bench.head_range(56, world, rank)
        total = bench.sum_over_ranks([nh, 1.0], world)
        seed = bench.rank_seed(1005, rank)
        seeds = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(seeds, torch.tensor([seed]))
        out[rank] = (got, [int(x) for x in seeds], (h0, nh), total)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timings_and_distinct_seeds():
    world = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        got, seeds, _, total = res[r]
        assert got == [11.0, 5.0, 1.0]
        assert seeds == [1005, 1006]
        assert total == [56.0, 2.0]  # the ranks' head shares add up to the whole call
    assert res[0][2] == (0, 28) and res[1][2] == (28, 28)


def test_whole_job_throughput_scales_with_ranks():
    one = bench.whole_job_tflops(51.9e12, 5, 1, 500.0)
    two = bench.whole_job_tflops(51.9e12, 5, 2, 500.0)
    assert one == pytest.approx(519.0) and two == pytest.approx(2 * one)
    assert bench.max_over_ranks([1.0, 2.0], 1) == [1.0, 2.0]


@pytest.mark.parametrize("H,world", [(56, 1), (56, 2), (56, 3), (56, 8), (7, 4), (5, 5)])
def test_head_ranges_cover_every_head_once(H, world):
    seen = []
    for r in range(world):
        h0, nh = bench.head_range(H, world, r)
        assert nh >= 1 and nh in (H // world, H // world + 1)
        seen.extend(range(h0, h0 + nh))
    assert seen == list(range(H))
