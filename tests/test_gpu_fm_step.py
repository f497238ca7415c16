"""GPU parity of wan_fm_step (fused CFG + Euler) against the fp64 oracle."""

import numpy as np
import pytest
import torch

from gpu_common import STEP_REL, cuda
from oracle import grid as ogrid
from oracle import schedule as osched
from oracle import step as ostep
from video_diffusion_transformer_self_b200 import build, inputs, wan
from video_diffusion_transformer_self_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _latent_numel(w):
    return int(np.prod(ogrid.latent_shape(w.frames, w.height, w.width)))


def _check_step(x_gpu, x_in, c, u, guide, s0, s1):
    got = x_gpu.double().cpu().numpy()
    want = ostep.fm_step(x_in.numpy(), c.numpy(),
                         None if u is None else u.numpy(), guide, s0, s1)
    # per element |err| <= 1e-6 (|x| + |dt| (|u| + |w| (|c| + |u|)))
    dt = abs(s1 - s0)
    cn = np.abs(c.numpy().astype(np.float64))
    un = 0.0 if u is None else np.abs(u.numpy().astype(np.float64))
    scale = np.abs(x_in.numpy().astype(np.float64)) + dt * (
        un + abs(guide) * (cn + un) + cn)
    err = np.abs(got - want)
    assert np.all(err <= STEP_REL * scale + 1e-30), float(np.max(err / scale))
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= STEP_REL, rel


@pytest.mark.parametrize("widx", [0, 1, 2, 3])
@pytest.mark.parametrize("cfg", [False, True])
def test_one_step_on_latent(widx, cfg):
    w = WORKLOADS[widx]
    n = _latent_numel(w)
    x = inputs.randn_f32((n,), inputs.seed_for(widx, "x"))
    c = inputs.randn_f32((n,), inputs.seed_for(widx, "v_cond"))
    u = inputs.randn_f32((n,), inputs.seed_for(widx, "v_uncond")) if cfg \
        else None
    sig = wan.fm_sigmas(w.steps, w.shift)
    guide = 4.0 if cfg else 1.0
    xg = cuda(x.clone())
    wan.fm_step(xg, cuda(c), None if u is None else cuda(u), guide, sig[0],
                sig[1])
    torch.cuda.synchronize()
    _check_step(xg, x, c, u, guide, sig[0], sig[1])


def test_literal_sigma_reading_tiny():
    # The tiny case read literally: sigma 1.0 -> 0.975.
    n = 2048
    x = inputs.randn_f32((n,), inputs.seed_for(0, "x"))
    c = inputs.randn_f32((n,), inputs.seed_for(0, "v_cond"))
    xg = cuda(x.clone())
    wan.fm_step(xg, cuda(c), None, 1.0, 1.0, 0.975)
    torch.cuda.synchronize()
    _check_step(xg, x, c, None, 1.0, 1.0, 0.975)


@pytest.mark.parametrize("n", [1, 3, 5, 4097, 1 << 20, (1 << 20) + 7])
def test_ragged_sizes(n):
    x = inputs.randn_f32((n,), 7)
    c = inputs.randn_f32((n,), 8)
    u = inputs.randn_f32((n,), 9)
    xg = cuda(x.clone())
    wan.fm_step(xg, cuda(c), cuda(u), 3.0, 0.7, 0.65)
    torch.cuda.synchronize()
    _check_step(xg, x, c, u, 3.0, 0.7, 0.65)


def test_no_write_past_end():
    n = 1001
    buf = torch.full((n + 64,), 123.0, device="cuda")
    x = buf[:n]
    c = cuda(inputs.randn_f32((n,), 11))
    wan.fm_step(x, c, None, 1.0, 1.0, 0.5)
    torch.cuda.synchronize()
    assert torch.all(buf[n:] == 123.0)


def test_zero_dt_identity_and_empty():
    x = cuda(inputs.randn_f32((999,), 12))
    x0 = x.clone()
    wan.fm_step(x, cuda(inputs.randn_f32((999,), 13)), None, 1.0, 0.5, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(x, x0)
    e = torch.empty(0, device="cuda")
    wan.fm_step(e, torch.empty(0, device="cuda"), None, 1.0, 1.0, 0.0)


def test_forty_step_loop_lands_on_x0():
    # 480p 165-frame latent, shift 12, 40 steps, constant seeded velocity
    # v = x1 - x0: Euler from x1 must land on x0 (rectified-flow closed form).
    w = WORKLOADS[4]
    n = _latent_numel(w)
    x0 = inputs.randn_f32((n,), inputs.seed_for(4, "x0"))
    x1 = inputs.randn_f32((n,), inputs.seed_for(4, "x"))
    v = x1 - x0
    sig = wan.fm_sigmas(40, 12.0)
    assert np.allclose(sig, osched.sigmas(40, 12.0), rtol=0, atol=1e-15)
    xg = cuda(x1.clone())
    vg = cuda(v)
    for i in range(40):
        wan.fm_step(xg, vg, None, 1.0, sig[i], sig[i + 1])
    torch.cuda.synchronize()
    got = xg.double().cpu().numpy()
    want = x0.numpy().astype(np.float64)
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    assert rel <= STEP_REL, rel
