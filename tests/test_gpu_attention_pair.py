"""GPU parity of wan_self_attn_pair (the CTA-pair self-attention kernel)
against the fp64 oracle: in full on small grids (less than one pair tile,
ragged tails, several key blocks, a batch of two), bit-for-bit against
itself under NaN guard bands, and on 4,096 sampled rows of every head at
the two token counts of the metric."""

import os

import numpy as np
import pytest
import torch

from gpu_common import (assert_attn_close, assert_heads_close, check_guards,
                        cuda, f64, guarded_empty_like, head_metrics,
                        map_threads, scale_for)
from oracle import attention as oattn
from oracle import grid as ogrid
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, wan
from video_diffusion_transformer_self_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _qkv(B, L, H, seed, q_scale=1.0):
    q = inputs.randn_bf16((B, L, H, 128), seed, q_scale)
    k = inputs.randn_bf16((B, L, H, 128), seed + 1)
    v = inputs.randn_bf16((B, L, H, 128), seed + 2)
    return q, k, v


def _run(q, k, v, grid):
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o, buf, guard = guarded_empty_like(qg)
    wan.self_attn_pair(qg, kg, vg, o, wan.grid(*grid))
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    return o


CASES = [
    ((2, 4, 4), 1, 2, 1.0),      # 32 tokens: less than one CTA's rows
    ((1, 1, 1), 1, 1, 1.0),      # a single token
    ((3, 7, 13), 2, 3, 1.0),     # 273 tokens: ragged, 2 key blocks + tail
    ((2, 8, 16), 1, 2, 1.0),     # 256 tokens: exactly one pair tile
    ((5, 10, 20), 1, 2, 1.0),    # 1,000 tokens: 8 key blocks (slot ring
                                 # wraps), ragged last tile
    ((5, 10, 20), 1, 1, 8.0),    # peaked softmax: max grows, O rescaled
    ((3, 9, 15), 2, 2, 1.0),     # 405 tokens, batch 2
]


@pytest.mark.parametrize("grid,B,H,qs", CASES)
def test_pair_matches_oracle(grid, B, H, qs):
    L = grid[0] * grid[1] * grid[2]
    q, k, v = _qkv(B, L, H, 4000 + L + B, qs)
    got = f64(_run(q, k, v, grid))
    want = oattn.attention(f64(q), f64(k), f64(v), scale_for())
    assert_attn_close(got, want, "pair L=%d B=%d H=%d q x%g" % (L, B, H, qs))


def test_pair_7800_full_and_equals_reference_kernel_layout():
    # 480p-17f: 7,800 tokens x 12 heads in full against the oracle
    w = WORKLOADS[1]
    grid = ogrid.token_grid(w.frames, w.height, w.width)
    L = ogrid.token_count(grid)
    q, k, v = _qkv(1, L, w.heads, inputs.seed_for(1, "q"))
    got = f64(_run(q, k, v, grid))

    def one(h):
        want = oattn.attention(f64(q[:, :, h:h + 1]), f64(k[:, :, h:h + 1]),
                               f64(v[:, :, h:h + 1]), scale_for(),
                               row_block=256)
        return head_metrics("pair 7800 h%d" % h, got[:, :, h:h + 1], want)

    assert_heads_close(map_threads(one, range(w.heads)), "pair 7800")


@pytest.mark.parametrize("grid,B,H", [((3, 7, 13), 2, 3), ((5, 10, 20), 1, 2),
                                      ((21, 6, 8), 1, 4)])
def test_pair_rotates_q_in_kernel(grid, B, H):
    # k rotated by the stand-alone pass (k alone), q in the kernel's tile
    # stage; compared with the oracle's rotation of both
    L = grid[0] * grid[1] * grid[2]
    q, k, v = _qkv(B, L, H, 5100 + L)
    g = wan.grid(*grid)
    table = wan.rope3d_table(g)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    wan.rope3d_qk(None, kg, g, table)
    o, buf, guard = guarded_empty_like(qg)
    wan.self_attn_pair(qg, kg, vg, o, g, table_q=table)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    check_guards(buf, guard)
    assert torch.equal(qg.cpu(), q)        # q in memory is untouched
    want = oattn.attention(orope.rope3d(f64(q), grid),
                           orope.rope3d(f64(k), grid), f64(v), scale_for())
    assert_attn_close(f64(o), want, "pair rope-q L=%d" % L)


def test_pair_deterministic():
    q, k, v = _qkv(1, 1000, 2, 77)
    a = _run(q, k, v, (5, 10, 20))
    b = _run(q, k, v, (5, 10, 20))
    assert torch.equal(a, b)


def _rows():
    return int(os.environ.get("WAN_PARITY_ROWS", 4096))


@pytest.mark.parametrize("widx", [2, 3])
def test_pair_full_size_sampled(widx):
    # the metric's token counts: 480p-81f (B 2 x 12 heads x 32,760) and
    # 720p-81f (B 1 x 40 x 75,600), Q / K pre-rotated by the RoPE pass
    w = WORKLOADS[widx]
    grid = ogrid.token_grid(w.frames, w.height, w.width)
    L = ogrid.token_count(grid)
    shape = (w.batch, L, w.heads, 128)
    q = inputs.randn_bf16(shape, inputs.seed_for(widx, "q"))
    k = inputs.randn_bf16(shape, inputs.seed_for(widx, "k"))
    v = inputs.randn_bf16(shape, inputs.seed_for(widx, "v"))
    g = wan.grid(*grid)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o = torch.empty_like(qg)
    wan.rope3d_qk(qg, kg, g, wan.rope3d_table(g))
    wan.self_attn_pair(qg, kg, vg, o, g)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    o = o.cpu()
    del qg, kg, vg
    angles = orope.token_angles(grid)

    def one(bh):
        b, h = bh
        rows = inputs.sample_rows(
            L, _rows(), inputs.seed_for(widx, "rows") + 1000 * b + h).numpy()
        qh = orope.apply_angles(f64(q[b:b + 1, rows, h:h + 1]), angles[rows])
        kh = orope.apply_angles(f64(k[b:b + 1, :, h:h + 1]), angles)
        want = oattn.attention(qh, kh, f64(v[b:b + 1, :, h:h + 1]),
                               scale_for(), row_block=128)
        return head_metrics("pair %s b%d h%d" % (w.name, b, h),
                            f64(o[b:b + 1, rows, h:h + 1]), want)

    assert_heads_close(map_threads(one, [(b, h) for b in range(w.batch)
                                         for h in range(w.heads)]),
                       "pair " + w.name)
