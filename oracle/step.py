"""CFG combine and Euler flow step in fp64 (oracle; test infrastructure only).

Wan2.2 source reading, ch. 1, section "From DDPM to flow matching": the path
is the straight line ``x_t = (1 - t) x0 + t x1`` with constant velocity
``dx/dt = x1 - x0``; the scheduler's clean estimate is
``x0_pred = sample - sigma * model_output`` and the page shows
``x_t - sigma v = x0``.

Wan2.2 source reading, ch. 5, section "UniPC": the plainest integrator is
Euler, taking the velocity constant over the step, ``x <- x - dsigma * v``
with sigma decreasing; written with the schedule's own values this is
``x <- x + (sigma_next - sigma) * v``.

Wan2.2 source reading, ch. 5, section "CFG": the guided velocity is
``uncond + w * (cond - uncond)``.
"""

import numpy as np


def cfg_combine(v_cond, v_uncond, guide):
    """uncond + guide * (cond - uncond) in fp64; v_uncond None -> cond."""
    c = np.asarray(v_cond, dtype=np.float64)
    if v_uncond is None:
        return c
    u = np.asarray(v_uncond, dtype=np.float64)
    return u + float(guide) * (c - u)


def euler_step(x, v, sigma, sigma_next):
    """x + (sigma_next - sigma) * v in fp64."""
    x = np.asarray(x, dtype=np.float64)
    return x + (float(sigma_next) - float(sigma)) * np.asarray(v, np.float64)


def fm_step(x, v_cond, v_uncond, guide, sigma, sigma_next):
    """One guided Euler step: the two functions above in sequence."""
    return euler_step(x, cfg_combine(v_cond, v_uncond, guide), sigma,
                      sigma_next)


def x0_estimate(sample, model_output, sigma):
    """Clean-sample estimate sample - sigma * model_output (fp64)."""
    return (np.asarray(sample, np.float64)
            - float(sigma) * np.asarray(model_output, np.float64))
