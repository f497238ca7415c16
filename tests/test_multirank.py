"""The benchmark's multi-rank host logic with two gloo ranks on the CPU:
each rank draws its own inputs, timings reduce to the slowest rank, and the
whole-job value counts every rank's work over that time."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from video_diffusion_transformer_self_b200 import inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # per-rank timings: the slowest rank decides
        ms = [10.0 + rank, 3.0 * (world - rank)]
        red = bench.max_over_ranks(ms, dist, "cpu")
        # per-rank inputs differ (independent problems, weak scaling)
        seed = inputs.seed_for(3, "q") + bench.rank_seed_offset(rank)
        x = inputs.randn_bf16((4, 8), seed).float()
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out[rank] = (red, [g.clone() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world,
                 join=True)
        res = dict(out)
    for rank in range(world):
        red, gathered = res[rank]
        assert red == [10.0 + world - 1, 3.0 * world]
        assert not torch.equal(gathered[0], gathered[1])
    assert bench.rank_seed_offset(0) == 0


def test_job_throughput_counts_all_ranks():
    one = bench.job_throughput(1, 1.17e14, 10, 1000.0)
    four = bench.job_throughput(4, 1.17e14, 10, 1000.0)
    assert four == pytest.approx(4 * one)
    assert one == pytest.approx(1170.0)  # 10 x 1.17e14 FLOP in 1 s
    assert bench.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]
