"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times: the whole attention call runs on the device; the oracle
evaluates seeded sampled query rows (always including the first and last
row, so the ragged tail tile is covered) against all keys.

Rows per (batch, head): WAN_PARITY_ROWS (default 256 at 75,600 and 65,520
tokens, 512 at 32,760 tokens)."""

import os

import numpy as np
import pytest
import torch

from gpu_common import assert_attn_close, cuda, f64, scale_for
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


def _rows(default):
    return int(os.environ.get("WAN_PARITY_ROWS", default))


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
    else:
        wan.self_attn(qg, kg, vg, o, g, table=table)
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    o = o.cpu()
    del qg, kg, vg
    worst = (0.0, 0.0)
    for b in range(w.batch):
        for h in range(w.heads):
            rows = inputs.sample_rows(
                L, n_rows, inputs.seed_for(widx, "rows") + 1000 * b + h).numpy()
            qh = orope.rope3d(f64(q[b:b + 1, :, h:h + 1]), grid)[:, rows]
            kh = orope.rope3d(f64(k[b:b + 1, :, h:h + 1]), grid)
            vh = f64(v[b:b + 1, :, h:h + 1])
            want = oattn.attention(qh, kh, vh, scale_for())
            got = f64(o[b:b + 1, rows, h:h + 1])
            ma, rf = assert_attn_close(got, want, "%s b%d h%d" % (w.name, b, h))
            worst = (max(worst[0], ma), max(worst[1], rf))
    return worst


def test_self_attn_480p_81f_sampled():
    _sampled_self_parity(2, _rows(512), "fused")


def test_self_attn_720p_81f_sampled():
    _sampled_self_parity(3, _rows(256), "fused")


def test_self_attn_720p_81f_prerotated_sampled():
    _sampled_self_parity(3, _rows(64), "pre")


def test_self_attn_480p_165f_sampled():
    _sampled_self_parity(4, _rows(64), "fused")


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
    rows = inputs.sample_rows(L, 2048, inputs.seed_for(widx, "rows")).numpy()
    want = oattn.attention(f64(q[:, rows]), f64(kc), f64(vc), scale_for(),
                           kv_lens=lens)
    got = f64(o[:, rows])
    assert_attn_close(got, want, "cross " + w.name)
