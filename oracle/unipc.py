"""UniPC (order 2) flow-matching sampler step in fp64 (oracle; test
infrastructure only).

Wan2.2 source reading, ch. 5, section "UniPC": Wan's default integrator is a
multistep predictor-corrector (``solver_order=2``).  The predictor fits the
trend of the model outputs of the last two steps and extrapolates to the next
stop; once the model has been evaluated there, the corrector revisits the
step just taken with that new output, at no extra forward; the local error
drops from Euler's first-order term to third order.  Ch. 1 ("From DDPM to
flow matching") fixes the path ``x = (1 - sigma) x0 + sigma noise`` and the
clean estimate ``x0_pred = sample - sigma * model_output``.

The pages give no coefficient, so the steps below follow the published UniPC
method (Zhao et al., "UniPC: A Unified Predictor-Corrector Framework for Fast
Sampling of Diffusion Models", 2023) in its data-prediction form, with the
coefficients solved exactly from its order conditions.  Readings taken
where the pages are silent:

* alpha = 1 - sigma and lambda = log(alpha / sigma), the half log-SNR of the
  straight path; lambda(1) = -inf and lambda(0) = +inf are taken as limits;
* the exact solution from sigma_s to sigma_t (t after s) is
  ``x_t = (sigma_t / sigma_s) x_s + alpha_t * sum_k D^k m(s) psi_k(h)``,
  h = lambda_t - lambda_s, ``psi_k(h) = int_0^h exp(tau - h) tau^k / k!
  dtau``; the update keeps the k = 0 term exactly and replaces the rest by
  sum_m c_m D_m / r_m over differences ``D_m = m(lambda_s + r_m h) - m(s)``,
  with c solving ``sum_m c_m r_m^(k-1) = k! psi_k(h) / h^k`` for k = 1 .. p
  (the paper's B(h) cancels out of an exactly solved system);
* predictor: order 2 (one earlier model output, r < 0) whenever an earlier
  output exists at finite lambda and the target sigma is not 0; otherwise
  order 1.  The step to sigma = 0 (lambda = +inf) must be first order: the
  order-2 term has no limit there (r -> 0);
* corrector: after the model output at the predicted sample is known, the
  step just taken is redone with the same earlier differences plus the new
  point (r = 1), i.e. one order higher; the model output is taken at the
  predicted sample and reused for the corrected one (no extra forward);
* an earlier point at sigma = 1 (lambda = -inf) is dropped: the limit of
  its coefficient times D / r is 0.

A first-order step reduces exactly to the Euler step of ``step.py``
(``x + (sigma_next - sigma) v``), which the pins use.
"""

import math

import numpy as np

from . import step as _step

SERIES_MAX_H = 1.0


def alpha(sigma):
    return 1.0 - float(sigma)


def log_snr(sigma):
    """lambda = log((1 - sigma) / sigma) with the limits at 0 and 1."""
    s = float(sigma)
    if not 0.0 <= s <= 1.0:
        raise ValueError("sigma must lie in [0, 1]")
    if s == 0.0:
        return math.inf
    if s == 1.0:
        return -math.inf
    return math.log((1.0 - s) / s)


def phi_q(k, h):
    """k! psi_k(h) / h^k, psi_k(h) = int_0^h exp(tau - h) tau^k / k! dtau.

    psi_k(h) = sum_{n>=0} (-1)^n h^(n+k+1) / (n+k+1)!; for h > 1 the
    recurrence psi_k = h^k / k! - psi_(k-1) (integration by parts), i.e.
    q_k = 1 - k q_(k-1) / h with q_0 = 1 - exp(-h); q_k(inf) = 1.
    """
    if h == math.inf:
        return 1.0
    if h <= 0.0:
        raise ValueError("h must be positive")
    if h <= SERIES_MAX_H:
        total = 0.0
        term = h / math.factorial(k + 1)  # n = 0: h^(k+1) / (k+1)! / h^k
        for n in range(40):
            total += term
            term *= -h / (n + k + 2)
        return math.factorial(k) * total
    q = -math.expm1(-h)
    for j in range(1, k + 1):
        q = 1.0 - j * q / h
    return q


def solve_coefficients(rs, h):
    """c with sum_m c_m r_m^(k-1) = q_k(h), k = 1 .. len(rs)."""
    p = len(rs)
    if p == 0:
        return np.zeros(0)
    R = np.array([[float(r) ** (k - 1) for r in rs] for k in range(1, p + 1)])
    g = np.array([phi_q(k, h) for k in range(1, p + 1)])
    return np.linalg.solve(R, g)


def exponential_update(x_s, sigma_s, sigma_t, m_s, diffs):
    """(sigma_t / sigma_s) x_s + alpha_t (q_0 m_s + sum c_m D_m / r_m).

    diffs: list of (D_m, r_m).  sigma_s > 0.
    """
    lam_s, lam_t = log_snr(sigma_s), log_snr(sigma_t)
    h = lam_t - lam_s
    rs = [r for _, r in diffs]
    c = solve_coefficients(rs, h)
    acc = phi_q(0, h) * np.asarray(m_s, np.float64)
    for cm, (D, r) in zip(c, diffs):
        acc = acc + (cm / r) * np.asarray(D, np.float64)
    return (float(sigma_t) / float(sigma_s)) * np.asarray(x_s, np.float64) \
        + alpha(sigma_t) * acc


def predictor_order(sigmas, i):
    """Order of the predictor that goes from sigma_i to sigma_(i+1)."""
    if i >= 1 and sigmas[i + 1] > 0.0 and math.isfinite(log_snr(sigmas[i - 1])):
        return 2
    return 1


def predictor(x_c, m, sigmas, i):
    """x~_(i+1) from the corrected sample x_c at sigma_i.

    m: dict step index -> data prediction (needs m[i], and m[i-1] at order 2).
    """
    diffs = []
    if predictor_order(sigmas, i) == 2:
        h = log_snr(sigmas[i + 1]) - log_snr(sigmas[i])
        r = (log_snr(sigmas[i - 1]) - log_snr(sigmas[i])) / h
        diffs.append((np.asarray(m[i - 1], np.float64) - m[i], r))
    return exponential_update(x_c, sigmas[i], sigmas[i + 1], m[i], diffs)


def corrector(x_c_prev, m, sigmas, i):
    """x^c_i: the step sigma_(i-1) -> sigma_i redone with the new m[i]."""
    diffs = []
    h = log_snr(sigmas[i]) - log_snr(sigmas[i - 1])
    if predictor_order(sigmas, i - 1) == 2:
        r = (log_snr(sigmas[i - 2]) - log_snr(sigmas[i - 1])) / h
        diffs.append((np.asarray(m[i - 2], np.float64) - m[i - 1], r))
    diffs.append((np.asarray(m[i], np.float64) - m[i - 1], 1.0))
    return exponential_update(x_c_prev, sigmas[i - 1], sigmas[i], m[i - 1],
                              diffs)


def unipc_step(x, x_c_prev, m_prev1, m_prev2, v_cond, v_uncond, guide,
               sigmas, i, use_corrector=True):
    """One sampler step at stop i (0 <= i < N) given the model output there.

    x: predicted sample x~_i; x_c_prev: corrected sample x^c_(i-1);
    m_prev1 / m_prev2: data predictions of stops i-1 / i-2 (None if absent).
    Returns (x~_(i+1), x^c_i, m_i).
    """
    n = len(sigmas) - 1
    if not 0 <= i < n:
        raise ValueError("step index out of range")
    v = _step.cfg_combine(v_cond, v_uncond, guide)
    m = {i: _step.x0_estimate(x, v, sigmas[i])}
    if m_prev1 is not None:
        m[i - 1] = np.asarray(m_prev1, np.float64)
    if m_prev2 is not None:
        m[i - 2] = np.asarray(m_prev2, np.float64)
    if i >= 1 and use_corrector:
        x_c = corrector(x_c_prev, m, sigmas, i)
    else:
        x_c = np.asarray(x, np.float64)
    x_next = predictor(x_c, m, sigmas, i)
    return x_next, x_c, m[i]


def unipc_sample(x_init, model, sigmas, use_corrector=True):
    """Run all N steps; model(x, sigma) -> velocity.  Returns x~_N."""
    x = np.asarray(x_init, np.float64)
    x_c = m1 = m2 = None
    for i in range(len(sigmas) - 1):
        v = model(x, sigmas[i])
        x, x_c, m = unipc_step(x, x_c, m1, m2, v, None, 1.0, sigmas, i,
                               use_corrector)
        m1, m2 = m, m1
    return x
