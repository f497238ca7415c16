"""GPU parity of wan_rope3d_qk (in-place 3D RoPE) against the fp64 oracle."""

import numpy as np
import pytest
import torch

from gpu_common import cuda
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _check(got_bf16, x_bf16, grid):
    x = x_bf16.double().numpy()
    want = orope.rope3d(x, grid)
    got = got_bf16.double().cpu().numpy()
    # bf16 output: half an ulp is <= 2^-8 of the value; fp32 arithmetic and
    # the fp32 table add ~1e-6 of the pair's norm.
    pair = np.sqrt(x[..., 0::2] ** 2 + x[..., 1::2] ** 2)
    pair = np.repeat(pair, 2, axis=-1)
    bound = 2.0 ** -8 * np.abs(want) + 1e-6 * pair + 1e-30
    err = np.abs(got - want)
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("grid,B,H", [((2, 4, 4), 1, 2), ((3, 7, 13), 2, 3),
                                      ((1, 1, 1), 1, 1), ((5, 30, 52), 1, 12),
                                      ((21, 45, 80), 1, 1)])
def test_rope_qk_matches_oracle(grid, B, H):
    L = grid[0] * grid[1] * grid[2]
    q = inputs.randn_bf16((B, L, H, 128), 21)
    k = inputs.randn_bf16((B, L, H, 128), 22)
    g = wan.grid(*grid)
    table = wan.rope3d_table(g)
    qg, kg = cuda(q), cuda(k)
    wan.rope3d_qk(qg, kg, g, table)
    torch.cuda.synchronize()
    _check(qg, q, grid)
    _check(kg, k, grid)


def test_rope_q_only_leaves_k():
    grid = (2, 3, 5)
    q = inputs.randn_bf16((1, 30, 2, 128), 23)
    k = inputs.randn_bf16((1, 30, 2, 128), 24)
    g = wan.grid(*grid)
    table = wan.rope3d_table(g)
    qg, kg = cuda(q), cuda(k)
    wan.rope3d_qk(qg, None, g, table)
    torch.cuda.synchronize()
    _check(qg, q, grid)
    assert torch.equal(kg.cpu(), k)


def test_table_values_match_oracle_angles():
    # Table entries are cos / sin of the oracle's per-band angles (fp32).
    grid = (4, 6, 9)
    g = wan.grid(*grid)
    tab = wan.rope3d_table(g).cpu().view(torch.float32).view(-1, 22, 2)
    tab = tab.double().numpy()
    wt, wh, ww = orope.band_widths(128)
    for band, (side, width, first, row0) in enumerate(
            [(4, wt, 0, 0), (6, wh, 0, 4), (9, ww, 1, 10)]):
        ang = orope.band_angles(np.arange(side), width)
        for pos in range(side):
            got = tab[row0 + pos, first:first + width // 2]
            assert np.max(np.abs(got[:, 0] - np.cos(ang[pos]))) < 1e-7
            assert np.max(np.abs(got[:, 1] - np.sin(ang[pos]))) < 1e-7
