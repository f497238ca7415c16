"""Pins of oracle/unipc.py against what the mathematics fixes.

* psi_k / phi_q against direct numerical quadrature of their definition;
* a first-order step is the Euler step (oracle/step.py, written separately
  from the pages' x <- x - dsigma v);
* exactness: the order-2 predictor integrates exactly when the data
  prediction is linear in lambda, the corrector when it is quadratic; the
  reference is the flow ODE dx/dsigma = (x - m) / sigma integrated by scipy
  (DOP853), not the exponential-integrator formula the oracle uses;
* measured global convergence orders on a nonlinear model: 2 for the
  predictor alone, 3 with the corrector (the pages: local error from first
  to third order);
* the step to sigma = 0 lands on the data prediction; sigma_0 = 1 is the
  limit of sigma_0 -> 1.
"""

import math

import numpy as np
import pytest
from scipy import integrate

from oracle import schedule, step, unipc


def psi_quad(k, h):
    f = lambda tau: math.exp(tau - h) * tau ** k / math.factorial(k)
    val, _ = integrate.quad(f, 0.0, h, epsabs=0, epsrel=1e-13, limit=200)
    return val


@pytest.mark.parametrize("k", [0, 1, 2, 3])
@pytest.mark.parametrize("h", [1e-3, 0.05, 0.4, 0.999, 1.001, 2.5, 9.0])
def test_phi_q_matches_quadrature(k, h):
    want = math.factorial(k) * psi_quad(k, h) / h ** k
    assert unipc.phi_q(k, h) == pytest.approx(want, rel=1e-10)


def test_phi_q_limits():
    for k in range(4):
        assert unipc.phi_q(k, math.inf) == 1.0
        # h -> 0: q_k ~ h / (k + 1)
        assert unipc.phi_q(k, 1e-8) == pytest.approx(1e-8 / (k + 1), rel=1e-6)
    assert unipc.phi_q(0, 0.7) == pytest.approx(1 - math.exp(-0.7), rel=1e-15)


def test_log_snr_limits():
    assert unipc.log_snr(0.5) == 0.0
    assert unipc.log_snr(0.0) == math.inf
    assert unipc.log_snr(1.0) == -math.inf
    assert unipc.log_snr(0.2) == pytest.approx(math.log(4.0))


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("shift,smax", [(12.0, 1.0), (5.0, 0.999), (1.0, 1.0)])
def test_first_step_is_euler(shift, smax):
    sig = schedule.sigmas(40, shift, smax)
    x, vc, vu = _rand(64, 1), _rand(64, 2), _rand(64, 3)
    x1, xc, m = unipc.unipc_step(x, None, None, None, vc, vu, 5.0, sig, 0)
    want = step.fm_step(x, vc, vu, 5.0, sig[0], sig[1])
    assert np.max(np.abs(x1 - want)) <= 1e-13 * np.max(np.abs(want))
    assert np.array_equal(xc, x)
    assert np.allclose(m, x - sig[0] * step.cfg_combine(vc, vu, 5.0),
                       rtol=0, atol=1e-15)


def test_last_step_lands_on_data_prediction():
    sig = schedule.sigmas(10, 12.0)
    n = len(sig) - 1
    x, xcp, m1, m2, v = (_rand(32, s) for s in range(5))
    x_next, _, m = unipc.unipc_step(x, xcp, m1, m2, v, None, 1.0, sig, n - 1)
    assert np.max(np.abs(x_next - (x - sig[n - 1] * v))) <= 1e-14
    assert np.array_equal(x_next, m)
    # ... which is the Euler step to sigma = 0 without the corrector's input
    assert np.allclose(x_next, step.euler_step(x, v, sig[n - 1], 0.0),
                       rtol=0, atol=1e-14)


def _ode_solution(x_s, sigma_s, sigma_t, m_of_lambda):
    """dx/dsigma = (x - m(lambda(sigma))) / sigma, integrated by DOP853."""
    def rhs(s, x):
        return (x - m_of_lambda(unipc.log_snr(s))) / s
    sol = integrate.solve_ivp(rhs, (sigma_s, sigma_t), np.asarray(x_s),
                              method="DOP853", rtol=1e-13, atol=1e-14)
    assert sol.success
    return sol.y[:, -1]


def test_ode_reference_is_exact_on_constant_prediction():
    # x = (1 - sigma) x0 + sigma eps is the solution when m = x0 everywhere
    x0, eps = _rand(8, 11), _rand(8, 12)
    got = _ode_solution(0.8 * eps + 0.2 * x0, 0.8, 0.3, lambda lam: x0)
    assert np.max(np.abs(got - (0.3 * eps + 0.7 * x0))) <= 1e-11


def test_predictor_exact_for_linear_prediction():
    a, b = _rand(16, 21), _rand(16, 22)
    m_of = lambda lam: a + b * lam
    sig = np.array([0.9, 0.7, 0.45, 0.2, 0.0])
    i = 1
    x_i = _rand(16, 23)
    m = {i - 1: m_of(unipc.log_snr(sig[i - 1])), i: m_of(unipc.log_snr(sig[i]))}
    assert unipc.predictor_order(sig, i) == 2
    got = unipc.predictor(x_i, m, sig, i)
    want = _ode_solution(x_i, sig[i], sig[i + 1], m_of)
    assert np.max(np.abs(got - want)) <= 1e-10 * np.max(np.abs(want))
    # a quadratic term is not integrated exactly by the predictor
    c = _rand(16, 24)
    m_of2 = lambda lam: a + b * lam + c * lam ** 2
    m2 = {k: m_of2(unipc.log_snr(sig[k])) for k in (i - 1, i)}
    err = np.max(np.abs(unipc.predictor(x_i, m2, sig, i)
                        - _ode_solution(x_i, sig[i], sig[i + 1], m_of2)))
    assert err > 1e-4


def test_corrector_exact_for_quadratic_prediction():
    a, b, c = _rand(16, 31), _rand(16, 32), _rand(16, 33)
    m_of = lambda lam: a + b * lam + c * lam ** 2
    sig = np.array([0.95, 0.8, 0.6, 0.35, 0.0])
    i = 2
    assert unipc.predictor_order(sig, i - 1) == 2
    x_prev = _rand(16, 34)
    m = {k: m_of(unipc.log_snr(sig[k])) for k in (i - 2, i - 1, i)}
    got = unipc.corrector(x_prev, m, sig, i)
    want = _ode_solution(x_prev, sig[i - 1], sig[i], m_of)
    assert np.max(np.abs(got - want)) <= 1e-10 * np.max(np.abs(want))
    # with only the new point (first corrector) a linear m is exact
    m_lin = lambda lam: a + b * lam
    ml = {k: m_lin(unipc.log_snr(sig[k])) for k in (0, 1)}
    got1 = unipc.corrector(x_prev, ml, sig, 1)
    want1 = _ode_solution(x_prev, sig[0], sig[1], m_lin)
    assert np.max(np.abs(got1 - want1)) <= 1e-10 * np.max(np.abs(want1))


def _nonlinear_model(x, sigma):
    # data prediction depends on x and on sigma: m = 0.5 tanh(x) + 0.3 cos(4 sigma)
    m = 0.5 * np.tanh(x) + 0.3 * np.cos(4.0 * sigma)
    return (x - m) / sigma  # velocity with x - sigma v = m


def _lambda_uniform_sigmas(n, s_hi=0.9, s_lo=0.1):
    lam = np.linspace(unipc.log_snr(s_hi), unipc.log_snr(s_lo), n + 1)
    return 1.0 / (1.0 + np.exp(lam))


def _global_error(n, use_corrector):
    sig = _lambda_uniform_sigmas(n)
    x0 = np.linspace(-2.0, 2.0, 9)
    got = unipc.unipc_sample(x0, _nonlinear_model, sig, use_corrector)
    sol = integrate.solve_ivp(lambda s, x: _nonlinear_model(x, s),
                              (sig[0], sig[-1]), x0, method="DOP853",
                              rtol=1e-13, atol=1e-14)
    return np.max(np.abs(got - sol.y[:, -1]))


def test_convergence_orders():
    e_p = [_global_error(n, False) for n in (10, 20, 40)]
    e_c = [_global_error(n, True) for n in (10, 20, 40)]
    order_p = math.log2(e_p[1] / e_p[2])
    order_c = math.log2(e_c[1] / e_c[2])
    assert 1.8 <= order_p <= 2.4, (e_p, order_p)
    assert 2.7 <= order_c <= 3.5, (e_c, order_c)
    assert e_c[2] < e_p[2]


def test_sigma_one_is_the_limit():
    # The dropped difference at lambda = -inf enters as D / r with
    # r ~ lambda_0 / h, so sigma_0 = 1 - delta approaches the sigma_0 = 1
    # result like 1 / log(1 / delta): the gap must shrink steadily.
    x0 = _rand(12, 41)
    s1 = schedule.sigmas(20, 5.0, 1.0)
    assert s1[0] == 1.0
    model = lambda x, s: _nonlinear_model(x, max(s, 1e-12))
    a = unipc.unipc_sample(x0, model, s1)
    assert np.all(np.isfinite(a))
    gaps = [np.max(np.abs(a - unipc.unipc_sample(
        x0, model, schedule.sigmas(20, 5.0, 1.0 - d)))) for d in
        (1e-3, 1e-6, 1e-10, 1e-15)]
    assert all(g1 > g2 for g1, g2 in zip(gaps, gaps[1:])), gaps
    assert gaps[-1] <= 2e-6


# ---- planted mistakes: each must break one of the pins above ------------

def _predictor_error():
    a, b = _rand(16, 21), _rand(16, 22)
    m_of = lambda lam: a + b * lam
    sig = np.array([0.9, 0.7, 0.45, 0.2, 0.0])
    x_i = _rand(16, 23)
    m = {k: m_of(unipc.log_snr(sig[k])) for k in (0, 1)}
    got = unipc.predictor(x_i, m, sig, 1)
    want = _ode_solution(x_i, sig[1], sig[2], m_of)
    return np.max(np.abs(got - want))


def _corrector_error():
    a, b, c = _rand(16, 31), _rand(16, 32), _rand(16, 33)
    m_of = lambda lam: a + b * lam + c * lam ** 2
    sig = np.array([0.95, 0.8, 0.6, 0.35, 0.0])
    x_prev = _rand(16, 34)
    m = {k: m_of(unipc.log_snr(sig[k])) for k in (0, 1, 2)}
    got = unipc.corrector(x_prev, m, sig, 2)
    want = _ode_solution(x_prev, sig[1], sig[2], m_of)
    return np.max(np.abs(got - want))


def test_pins_hold_unplanted():
    assert _predictor_error() < 1e-9
    assert _corrector_error() < 1e-9


def test_planted_phi_order_mistake_is_caught(monkeypatch):
    right = unipc.phi_q
    monkeypatch.setattr(unipc, "phi_q", lambda k, h: right(k + 1, h)
                        if k >= 1 else right(k, h))
    assert _predictor_error() > 1e-4


def test_planted_dropped_new_point_is_caught(monkeypatch):
    right = unipc.exponential_update

    def drop_last(x_s, sigma_s, sigma_t, m_s, diffs):
        return right(x_s, sigma_s, sigma_t, m_s, diffs[:-1])
    monkeypatch.setattr(unipc, "exponential_update", drop_last)
    assert _corrector_error() > 1e-4


def test_planted_clean_estimate_sign_is_caught(monkeypatch):
    monkeypatch.setattr(unipc._step, "x0_estimate",
                        lambda x, v, s: np.asarray(x, np.float64)
                        + float(s) * np.asarray(v, np.float64))
    sig = schedule.sigmas(40, 12.0)
    x, vc = _rand(64, 1), _rand(64, 2)
    x1, _, _ = unipc.unipc_step(x, None, None, None, vc, None, 1.0, sig, 0)
    want = step.fm_step(x, vc, None, 1.0, sig[0], sig[1])
    assert np.max(np.abs(x1 - want)) > 1e-3
