"""Ulysses exchange logic with gloo ranks on the CPU (no GPU).

The product module ``ulysses`` moves layouts with the library's CUDA
transpose and attends with the CUDA kernel; here both are replaced by plain
CPU stand-ins (a torch transpose of the same documented layout, and the fp64
oracle attention), so that what is tested is the host logic: which chunk
goes to which rank, the two all-to-alls per direction, the padding rule.
Each rank's output must equal the oracle on the whole, unsharded problem.
"""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import attention as oattn
from video_diffusion_transformer_self_b200 import inputs, ulysses, wan


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cpu_swap(inp, out, a, b, row_bytes):
    # out[j][i][:] = inp[i][j][:], rows of row_bytes
    n = row_bytes // inp.element_size()
    src = inp.reshape(-1)[: a * b * n].view(a, b, n)
    out.reshape(-1)[: a * b * n].copy_(src.transpose(0, 1).reshape(-1))


def _oracle_attention(q, k, v, o, g, table, scale):
    assert table is None
    if scale is None:  # the library's default, 1 / sqrt(head_dim)
        scale = 1 / math.sqrt(q.shape[-1])
    o.copy_(torch.from_numpy(oattn.attention(
        q.double().numpy(), k.double().numpy(), v.double().numpy(),
        scale)).to(o.dtype))


def _full_inputs(B, Lpad, H, seed):
    d = 128
    def r(role):
        return inputs.randn_f32((B, Lpad, H, d), inputs.seed_for(seed, role))
    return r("q"), r("k"), r("v")


def _worker(rank, world, port, cases, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ulysses._swap = _cpu_swap
    ulysses._attention = _oracle_attention
    try:
        res = []
        for (B, grid, H, seed) in cases:
            L = grid[0] * grid[1] * grid[2]
            Lpad = ulysses.padded_len(L, world)
            Ls = Lpad // world
            q, k, v = _full_inputs(B, Lpad, H, seed)
            sl = slice(rank * Ls, (rank + 1) * Ls)
            o = ulysses.ulysses_self_attn(
                q[:, sl].contiguous(), k[:, sl].contiguous(),
                v[:, sl].contiguous(), wan.grid(*grid),
                softmax_scale=1 / math.sqrt(128))
            res.append(o.clone())
        out[rank] = res
    finally:
        dist.destroy_process_group()


CASES = [(1, (2, 3, 5), 4, 0),   # L 30, even split
         (2, (2, 3, 5), 6, 1),   # batch 2
         (1, (3, 3, 3), 2, 2)]   # L 27: padded to 28 on 2 ranks


@pytest.mark.parametrize("world", [2])
def test_ulysses_two_gloo_ranks(world):
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, _free_port(), CASES, out),
                 nprocs=world, join=True)
        res = dict(out)
    for ci, (B, grid, H, seed) in enumerate(CASES):
        L = grid[0] * grid[1] * grid[2]
        Lpad = ulysses.padded_len(L, world)
        Ls = Lpad // world
        q, k, v = _full_inputs(B, Lpad, H, seed)
        want = oattn.attention(q[:, :L].double().numpy(),
                               k[:, :L].double().numpy(),
                               v[:, :L].double().numpy(), 1 / math.sqrt(128))
        got = torch.cat([res[r][ci] for r in range(world)], dim=1)
        assert got.shape == (B, Lpad, H, 128)
        # fp32 storage of an fp64 result: the exchange itself moves bits
        np.testing.assert_allclose(got[:, :L].double().numpy(), want,
                                   rtol=0, atol=2e-6 * np.abs(want).max())


def test_layout_helpers_are_inverse():
    # pack -> emulated exchange -> unpack, rank by rank, in one process
    P, B, Ls, H, d = 4, 2, 3, 8, 128
    xs = [torch.randn(B, Ls, H, d) for _ in range(P)]
    orig = ulysses._swap
    ulysses._swap = _cpu_swap
    try:
        sends = [ulysses.pack_seq_to_head(x, P) for x in xs]
        heads = [ulysses.unpack_seq_to_head(
            torch.stack([sends[src][dst] for src in range(P)]))
            for dst in range(P)]
        full = torch.cat(xs, dim=1)
        for r in range(P):
            assert torch.equal(heads[r], full[:, :, r * 2:(r + 1) * 2])
        back = [ulysses.pack_head_to_seq(h, P) for h in heads]
        seqs = [ulysses.unpack_head_to_seq(
            torch.stack([back[src][dst] for src in range(P)]))
            for dst in range(P)]
        for r in range(P):
            assert torch.equal(seqs[r], xs[r])
    finally:
        ulysses._swap = orig


def test_rejects_bad_splits():
    assert ulysses.padded_len(75601, 8) == 75608
    assert ulysses.padded_len(75600, 8) == 75600
    with pytest.raises(ValueError):
        ulysses.pack_seq_to_head(torch.zeros(1, 2, 6, 128), 4)  # 6 % 4
    with pytest.raises(ValueError):
        ulysses.pack_head_to_seq(torch.zeros(1, 6, 2, 128), 4)  # 6 % 4


# ---- bench.py --parallel ulysses: its host logic on two gloo ranks, with
# the same CPU stand-ins for the two kernels.

def _bench_worker(rank, world, port, out):
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ulysses._swap = _cpu_swap
    ulysses._attention = _oracle_attention
    try:
        grid, B, H = (3, 3, 3), 1, 4          # 27 tokens -> 28 on 2 ranks
        L = 27
        plan = bench.ulysses_plan(L, world, rank)
        q, k, v = _full_inputs(B, plan["Lpad"], H, 5)
        sl = slice(plan["first"], plan["end"])
        tags = []
        o = bench.ulysses_steps(q[:, sl].contiguous(), k[:, sl].contiguous(),
                                v[:, sl].contiguous(), wan.grid(*grid), None,
                                "pre", 2, mark=tags.append)
        red = bench.max_over_ranks([1.0 + rank, 5.0 - rank], dist, "cpu")
        out[rank] = (plan, o.clone(), tags, red)
    finally:
        dist.destroy_process_group()


def test_bench_ulysses_mode_two_gloo_ranks():
    import bench
    world = 2
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_bench_worker, args=(world, _free_port(), out),
                 nprocs=world, join=True)
        res = dict(out)
    plans = [res[r][0] for r in range(world)]
    # equal shards covering the padded sequence, in rank order
    assert [p["Ls"] for p in plans] == [14, 14]
    assert plans[0]["first"] == 0 and plans[1]["first"] == 14
    assert plans[1]["end"] == plans[0]["Lpad"] == 28
    # phases marked in order, once per step
    assert res[0][2] == ["start", "exchanged", "attended", "end"] * 2
    # timings reduce to the slowest rank
    assert res[0][3] == res[1][3] == [2.0, 5.0]
    q, k, v = _full_inputs(1, 28, 4, 5)
    want = oattn.attention(q[:, :27].double().numpy(),
                           k[:, :27].double().numpy(),
                           v[:, :27].double().numpy(), 1 / math.sqrt(128))
    got = torch.cat([res[r][1] for r in range(world)], dim=1)[:, :27]
    np.testing.assert_allclose(got.double().numpy(), want, rtol=0,
                               atol=2e-6 * np.abs(want).max())
    # strong scaling: one problem's FLOPs, not one per rank
    assert bench.ulysses_value(1, 40, 75600, 10, 1000.0) == pytest.approx(
        4.0 * 40 * 75600 ** 2 * 128 * 10 / 1e12)
