"""Full-size parity of the HBM passes in the launch configuration bench.py
times (720p-81f: 75,600 tokens x 40 heads, model dim 5,120), checked on
seeded sampled tokens against the fp64 oracle; the Ulysses pack of the
full Q is checked bit for bit on sampled rows."""

import numpy as np
import pytest
import torch

from gpu_common import cuda
from oracle import block as oblock
from oracle import rope as orope
from test_gpu_block import _bf16_bound
from video_diffusion_transformer_self_b200 import build, inputs, wan

pytestmark = pytest.mark.gpu

GRID = (21, 45, 80)
L, H, D = 75600, 40, 5120
N_SAMPLE = 2048


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _sample(seed):
    idx = inputs.sample_rows(L, N_SAMPLE, seed)
    return np.asarray(idx, dtype=np.int64)


def test_qk_norm_rope_720p_sampled():
    q = inputs.randn_bf16((1, L, H, 128), inputs.seed_for(3, "q"), 2.0)
    w = inputs.randn_f32((H * 128,), inputs.seed_for(3, "x"))
    g = wan.grid(*GRID)
    qg = cuda(q)
    wan.qk_norm_rope(qg, None, cuda(w), None, g, wan.rope3d_table(g))
    torch.cuda.synchronize()
    idx = _sample(51)
    x = q[0, idx].double().numpy().reshape(len(idx), H * 128)
    y = oblock.rms_norm(x, w.numpy()).reshape(len(idx), H, 128)
    want = orope.apply_angles(y, orope.token_angles(GRID)[idx])
    got = qg[0, torch.from_numpy(idx).cuda()].double().cpu().numpy()
    _bf16_bound(got, want,
                1e-5 * (1 + np.abs(want)).max(axis=-1, keepdims=True))


def test_adaln_and_gated_residual_720p_sampled():
    x = inputs.randn_f32((1, L, D), inputs.seed_for(3, "x"), 3.0)
    shift = inputs.randn_f32((1, D), 61, 0.2)
    scale = inputs.randn_f32((1, D), 62, 0.2)
    gate = inputs.randn_f32((1, D), 63, 0.5)
    xg = cuda(x)
    out = torch.empty((1, L, D), dtype=torch.bfloat16, device="cuda")
    wan.adaln_modulate(xg, cuda(shift), cuda(scale), out)
    wan.gated_residual(xg, out, cuda(gate))
    torch.cuda.synchronize()
    idx = _sample(52)
    ti = torch.from_numpy(idx).cuda()
    xs = x[0, idx].double().numpy()[None]
    want_m = oblock.adaln_modulate(xs, shift.double().numpy(),
                                   scale.double().numpy())
    got_m = out[0, ti].double().cpu().numpy()[None]
    _bf16_bound(got_m, want_m, 1e-5 * (1 + np.abs(want_m)))
    # the residual uses the bf16 modulated rows the kernel wrote
    want_r = oblock.gated_residual(xs, got_m, gate.double().numpy())
    got_r = xg[0, ti].double().cpu().numpy()[None]
    err = np.abs(got_r - want_r)
    assert np.all(err <= 1e-6 * (np.abs(xs) + np.abs(got_m * gate.numpy()))
                  + 1e-30), float(np.max(err))


def test_ulysses_pack_720p_sampled_rows():
    q = inputs.randn_bf16((1, L, H, 128), inputs.seed_for(3, "k"))
    P = 8
    qg = cuda(q)
    send = torch.empty_like(qg)
    row = (H // P) * 128 * 2
    wan.transpose_blocks(qg, send, L, P, row)
    torch.cuda.synchronize()
    sv = send.view(P, L, H // P, 128)
    idx = _sample(53)
    ti = torch.from_numpy(idx).cuda()
    for p in range(P):
        want = q[0, idx, p * (H // P):(p + 1) * (H // P)]
        assert torch.equal(sv[p, ti].cpu(), want), p
