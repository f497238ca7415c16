"""GPU parity of wan_unipc_step (fused CFG + UniPC corrector + predictor)
against the fp64 oracle, per stop and over a whole 40-step run."""

import numpy as np
import pytest
import torch

from gpu_common import cuda
from oracle import grid as ogrid
from oracle import schedule as osched
from oracle import unipc as ounipc
from test_unipc_host import oracle_coeffs
from video_diffusion_transformer_self_b200 import build, inputs, wan
from video_diffusion_transformer_self_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

# Each output is a short fp32 FMA chain over inputs and fp32-rounded
# coefficients: at most 4 roundings per term (coefficient, product, sum).
# Budget per term: 8 u, u = 2^-24 (twice that count).
TERM = 8.0 * 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    wan.lib()


def _numel(widx):
    w = WORKLOADS[widx]
    return int(np.prod(ogrid.latent_shape(w.frames, w.height, w.width)))


def _bounds(c, sigma, x, xc, m1, m2, vc, vu, w):
    """Per-element error bounds of (x~_(i+1), x^c_i, m_i)."""
    a = np.abs
    V = a(vc) if vu is None else a(vu) + abs(w) * (a(vc) + a(vu))
    m_abs = a(x) + sigma * V
    em = TERM * m_abs
    if c["corr_order"] == 0:
        xc_abs, exc = a(x), 0.0
    else:
        xc_abs = (abs(c["cx"]) * a(xc) + abs(c["cm1"]) * a(m1)
                  + abs(c["cm2"]) * a(m2) + abs(c["cm"]) * m_abs)
        exc = TERM * xc_abs + abs(c["cm"]) * em
    ex = (TERM * (abs(c["px"]) * xc_abs + abs(c["pm"]) * m_abs
                  + abs(c["pm1"]) * a(m1))
          + abs(c["px"]) * exc + abs(c["pm"]) * em)
    return ex, exc, em


def _inputs(widx, n):
    def r(role):
        return inputs.randn_f32((n,), inputs.seed_for(widx, role))
    return r("x"), r("x_corr"), r("m_prev1"), r("m_prev2"), r("v_cond"), \
        r("v_uncond")


def _run_stop(widx, n, sig, i, cfg, alias):
    x, xc, m1, m2, vc, vu = _inputs(widx, n)
    guide = 5.0 if cfg else 1.0
    c = wan.unipc_coeffs(sig, i)
    need_m1 = c["corr_order"] >= 1
    need_m2 = c["corr_order"] == 2
    xg, xcg = cuda(x.clone()), cuda(xc.clone())
    m1g = cuda(m1) if need_m1 else None
    m2g = cuda(m2.clone()) if need_m2 else None
    mo = m2g if (alias and need_m2) else torch.empty(n, device="cuda")
    wan.unipc_step(xg, xcg, m1g, m2g, mo, cuda(vc), cuda(vu) if cfg else None,
                   guide, sig, i)
    torch.cuda.synchronize()
    f = lambda t: t.numpy().astype(np.float64)
    want = ounipc.unipc_step(f(x), f(xc), f(m1) if need_m1 else None,
                             f(m2) if need_m2 else None, f(vc),
                             f(vu) if cfg else None, guide, sig, i)
    bounds = _bounds(c, sig[i], f(x), f(xc), f(m1), f(m2), f(vc),
                     f(vu) if cfg else None, guide)
    for name, g, w, b in zip(("x_next", "x_corr", "m"), (xg, xcg, mo),
                             want, bounds):
        got = g.double().cpu().numpy()
        err = np.abs(got - w)
        assert np.all(err <= b + 1e-37), (name, float(np.max(err - b)))
    return c


@pytest.mark.parametrize("i", [0, 1, 2, 3, 20, 38, 39])
@pytest.mark.parametrize("cfg", [False, True])
def test_stop_matches_oracle(i, cfg):
    sig = osched.sigmas(40, 12.0)
    n = _numel(1) + 3  # 480p-17f latent plus a ragged tail
    _run_stop(1, n, sig, i, cfg, alias=False)


@pytest.mark.parametrize("smax", [1.0, 0.999])
def test_every_stop_small(smax):
    sig = osched.sigmas(40, 12.0, smax)
    for i in range(40):
        _run_stop(0, _numel(0) + 1, sig, i, cfg=True, alias=True)


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 7, 4099])
def test_sizes_and_alias(n):
    sig = osched.sigmas(10, 5.0)
    for i in (0, 1, 4, 9):
        _run_stop(2, n, sig, i, cfg=True, alias=True)


def test_full_latent_720p_order2_stop():
    sig = osched.sigmas(40, 12.0)
    c = _run_stop(3, _numel(3), sig, 20, cfg=True, alias=True)
    assert c["corr_order"] == 2 and c["pred_order"] == 2


def test_forty_step_run():
    # The "model" is a fixed seeded velocity per stop, so both sides see the
    # same inputs and the run is a pure test of the sampler arithmetic.
    n = _numel(1)
    sig = osched.sigmas(40, 12.0)
    vs = [inputs.randn_f32((n,), inputs.seed_for(1, "v_cond") * 64 + i)
          for i in range(40)]
    x0 = inputs.randn_f32((n,), inputs.seed_for(1, "x"))
    x, xc = cuda(x0.clone()), torch.empty(n, device="cuda")
    bufs = [torch.empty(n, device="cuda"), torch.empty(n, device="cuda")]
    m1 = m2 = None
    for i in range(40):
        mo = bufs[0] if m1 is not bufs[0] else bufs[1]
        wan.unipc_step(x, xc, m1, m2, mo, cuda(vs[i]), None, 1.0, sig, i)
        m1, m2 = mo, m1
    torch.cuda.synchronize()
    assert wan.device_status() == 0
    model = lambda xx, s, _it=iter(vs): next(_it).numpy().astype(np.float64)
    want = ounipc.unipc_sample(x0.numpy().astype(np.float64), model, sig)
    got = x.double().cpu().numpy()
    rel = np.linalg.norm(got - want) / np.linalg.norm(want)
    # 40 stops of per-stop relative error <= ~8 u * sum|coef| (sum <= 3)
    assert rel <= 40 * 3 * TERM, rel
