"""Pins of the oracle's Euler / CFG step to the rectified-flow closed form."""

import numpy as np
import pytest

from oracle import schedule, step


def _rng(seed):
    return np.random.default_rng(seed)


@pytest.mark.parametrize("n_steps,shift", [(1, 5.0), (40, 12.0), (7, 1.0),
                                           (40, 5.0)])
def test_euler_lands_on_x0(n_steps, shift):
    # Straight path x_sigma = x0 + sigma (x1 - x0) with constant velocity:
    # Euler from sigma_0 = 1 (x = x1) to sigma_N = 0 lands on x0 for any
    # schedule, because the steps telescope.
    r = _rng(1)
    x0 = r.standard_normal(1000)
    x1 = r.standard_normal(1000)
    v = x1 - x0
    sig = schedule.sigmas(n_steps, shift)
    x = x1.copy()
    for i in range(n_steps):
        x = step.fm_step(x, v, None, 1.0, sig[i], sig[i + 1])
    assert np.max(np.abs(x - x0)) < 1e-12


def test_intermediate_points_on_line():
    r = _rng(2)
    x0, x1 = r.standard_normal(64), r.standard_normal(64)
    sig = schedule.sigmas(40, 12.0)
    x = x1.copy()
    for i in range(40):
        x = step.euler_step(x, x1 - x0, sig[i], sig[i + 1])
        want = (1 - sig[i + 1]) * x0 + sig[i + 1] * x1
        assert np.max(np.abs(x - want)) < 1e-12


def test_x0_identity():
    # x_t - sigma v = x0 for x_t = (1 - sigma) x0 + sigma x1, v = x1 - x0.
    r = _rng(3)
    x0, x1 = r.standard_normal(128), r.standard_normal(128)
    for sigma in (0.0, 0.3, 0.875, 1.0):
        xt = (1 - sigma) * x0 + sigma * x1
        assert np.max(np.abs(step.x0_estimate(xt, x1 - x0, sigma) - x0)) \
            < 1e-14


def test_cfg_special_cases():
    r = _rng(4)
    c, u = r.standard_normal(256), r.standard_normal(256)
    # u + 1 * (c - u) equals c up to one fp64 rounding of the difference
    assert np.max(np.abs(step.cfg_combine(c, u, 1.0) - c)) < 1e-14
    assert np.array_equal(step.cfg_combine(c, u, 0.0), u)
    assert np.array_equal(step.cfg_combine(c, None, 7.0), c)
    # linear in w: w = 2 is the reflection of uncond through cond
    assert np.allclose(step.cfg_combine(c, u, 2.0), 2 * c - u, rtol=0,
                       atol=1e-15)


def test_zero_dt_is_identity():
    r = _rng(5)
    x, v = r.standard_normal(99), r.standard_normal(99)
    assert np.array_equal(step.euler_step(x, v, 0.5, 0.5), x)


def test_step_direction():
    # sigma decreases, so the step moves against v
    x = np.zeros(4)
    v = np.ones(4)
    out = step.euler_step(x, v, 1.0, 0.9)
    assert np.all(out < 0)


def test_planted_sign_mistake_is_caught(monkeypatch):
    # A flipped dt sign must break the closed form pin.
    def wrong(x, v, sigma, sigma_next):
        return np.asarray(x, np.float64) + (sigma - sigma_next) * np.asarray(v)
    monkeypatch.setattr(step, "euler_step", wrong)
    r = _rng(6)
    x0, x1 = r.standard_normal(10), r.standard_normal(10)
    sig = schedule.sigmas(5, 3.0)
    x = x1.copy()
    for i in range(5):
        x = step.fm_step(x, x1 - x0, None, 1.0, sig[i], sig[i + 1])
    assert np.max(np.abs(x - x0)) > 0.1
