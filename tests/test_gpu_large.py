"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: the whole attention call runs on the device; the oracle
evaluates 4,096 seeded sampled query rows of every (batch row, head)
(always including the first and last row, so the ragged tail tile is
covered) against all keys, in fp64.

Heads are independent, so the oracle runs them on a thread pool.  Rows per
(batch, head): WAN_PARITY_ROWS (default 4096)."""

import os

import numpy as np
import pytest
import torch

from gpu_common import (assert_attn_close, assert_heads_close, cuda, f64,
                        head_metrics, map_threads, scale_for)
from oracle import attention as oattn
from oracle import grid as ogrid
from oracle import rope as orope
from video_diffusion_transformer_self_b200 import build, inputs, wan
from video_diffusion_transformer_self_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

ROW_BLOCK = 128  # oracle rows per matmul: bounds each thread's memory


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _rows():
    return int(os.environ.get("WAN_PARITY_ROWS", 4096))


def _workload_tensors(w):
    grid = ogrid.token_grid(w.frames, w.height, w.width)
    L = ogrid.token_count(grid)
    shape = (w.batch, L, w.heads, 128)
    q = inputs.randn_bf16(shape, inputs.seed_for(w.index, "q"))
    k = inputs.randn_bf16(shape, inputs.seed_for(w.index, "k"))
    v = inputs.randn_bf16(shape, inputs.seed_for(w.index, "v"))
    return grid, L, q, k, v


def _sampled_self_parity(widx, n_rows, mode):
    w = WORKLOADS[widx]
    grid, L, q, k, v = _workload_tensors(w)
    g = wan.grid(*grid)
    qg, kg, vg = cuda(q), cuda(k), cuda(v)
    o = torch.empty_like(qg)
    table = wan.rope3d_table(g)
    if mode == "pre":
        wan.rope3d_qk(qg, kg, g, table)
        wan.self_attn(qg, kg, vg, o, g)
    elif mode == "rope_q":
        wan.rope3d_qk(None, kg, g, table)
        wan.self_attn_rope_q(qg, kg, vg, o, g, table)
    else:
        wan.self_attn(qg, kg, vg, o, g, table=table)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    o = o.cpu()
    del qg, kg, vg
    angles = orope.token_angles(grid)

    def one(bh):
        b, h = bh
        rows = inputs.sample_rows(
            L, n_rows, inputs.seed_for(widx, "rows") + 1000 * b + h).numpy()
        qh = orope.apply_angles(f64(q[b:b + 1, rows, h:h + 1]), angles[rows])
        kh = orope.apply_angles(f64(k[b:b + 1, :, h:h + 1]), angles)
        vh = f64(v[b:b + 1, :, h:h + 1])
        want = oattn.attention(qh, kh, vh, scale_for(), row_block=ROW_BLOCK)
        got = f64(o[b:b + 1, rows, h:h + 1])
        return head_metrics("%s %s b%d h%d (%d rows)"
                            % (w.name, mode, b, h, len(rows)), got, want)

    res = map_threads(one, [(b, h) for b in range(w.batch)
                            for h in range(w.heads)])
    return assert_heads_close(res, "%s %s" % (w.name, mode))


def test_self_attn_480p_81f_sampled():
    _sampled_self_parity(2, _rows(), "fused")


def test_self_attn_480p_81f_prerotated_sampled():
    _sampled_self_parity(2, _rows(), "pre")


def test_self_attn_720p_81f_sampled():
    _sampled_self_parity(3, _rows(), "fused")


def test_self_attn_720p_81f_prerotated_sampled():
    _sampled_self_parity(3, _rows(), "pre")


def test_self_attn_720p_81f_rope_q_sampled():
    _sampled_self_parity(3, _rows(), "rope_q")


def test_self_attn_480p_165f_sampled():
    _sampled_self_parity(4, _rows(), "fused")


@pytest.mark.parametrize("widx", [2, 3])
def test_cross_attn_full_size(widx):
    w = WORKLOADS[widx]
    grid = ogrid.token_grid(w.frames, w.height, w.width)
    L = ogrid.token_count(grid)
    lens = inputs.uniform_int(w.batch, w.text_len_lo, w.text_len_hi,
                              inputs.seed_for(widx, "lens")).tolist()
    q = inputs.randn_bf16((w.batch, L, w.heads, 128),
                          inputs.seed_for(widx, "q"))
    kc = inputs.poison_tail(inputs.randn_bf16(
        (w.batch, w.text_tokens, w.heads, 128),
        inputs.seed_for(widx, "k_ctx")), lens)
    vc = inputs.poison_tail(inputs.randn_bf16(
        (w.batch, w.text_tokens, w.heads, 128),
        inputs.seed_for(widx, "v_ctx")), lens)
    qg = cuda(q)
    o = torch.empty_like(qg)
    wan.cross_attn(qg, cuda(kc), cuda(vc), o, lens)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    o = o.cpu()
    rows = inputs.sample_rows(L, _rows(), inputs.seed_for(widx, "rows")).numpy()

    def one(bh):
        b, h = bh
        want = oattn.attention(f64(q[b:b + 1, rows, h:h + 1]),
                               f64(kc[b:b + 1, :, h:h + 1]),
                               f64(vc[b:b + 1, :, h:h + 1]), scale_for(),
                               kv_lens=[lens[b]], row_block=ROW_BLOCK)
        got = f64(o[b:b + 1, rows, h:h + 1])
        return head_metrics("cross %s b%d h%d len %d" % (w.name, b, h,
                                                         lens[b]), got, want)

    res = map_threads(one, [(b, h) for b in range(w.batch)
                            for h in range(w.heads)])
    assert_heads_close(res, "cross " + w.name)
