"""Shifted sigma schedule in fp64 (oracle; test infrastructure only).

Wan2.2 source reading, ch. 1, section "One ruler, two scales": sigma lies in
[0, 1], the code's timestep is ``t = 1000 * sigma`` (``num_train_timesteps =
1000``), larger t is closer to noise.

Wan2.2 source reading, ch. 5, section "shift: where to put the 40 stops":
``set_timesteps`` first lays the points uniformly and then applies
``sigma = shift * s / (1 + (shift - 1) * s)``; with shift 12 and 40 steps
half of the points fall at t > 926 and the first timesteps (printed as
integers) are 999, 997, 995, 993, 990, 988.  Ch. 6 ("boundary and shift"):
with boundary 0.875, 26 of the 40 steps have t >= 875 and 14 fall below.

Readings taken where the page is silent:

* "laid uniformly" is s_i = s_max * (1 - i / N) for i = 0 .. N-1, with
  s_max = 1 by default; the printed list is reproduced with s_max = 0.999
  and integer truncation of t (``timesteps_int``);
* the schedule is closed by sigma_N = 0 so that the last Euler step lands on
  the clean sample (ch. 1: the sampler integrates back to x0).
"""

import numpy as np

NUM_TRAIN_TIMESTEPS = 1000


def shift_sigma(s, shift):
    """sigma = shift * s / (1 + (shift - 1) * s), elementwise in fp64."""
    s = np.asarray(s, dtype=np.float64)
    return shift * s / (1.0 + (shift - 1.0) * s)


def sigmas(n_steps, shift, s_max=1.0):
    """sigma_0 .. sigma_N (N + 1 values), sigma_N = 0."""
    if n_steps < 1:
        raise ValueError("n_steps must be >= 1")
    i = np.arange(n_steps, dtype=np.float64)
    s = s_max * (1.0 - i / n_steps)
    return np.concatenate([shift_sigma(s, shift), [0.0]])


def timesteps(n_steps, shift, s_max=1.0):
    """t_i = 1000 * sigma_i for the N sampling points (fp64)."""
    return NUM_TRAIN_TIMESTEPS * sigmas(n_steps, shift, s_max)[:n_steps]


def timesteps_int(n_steps, shift, s_max=1.0):
    """Integer timesteps by truncation toward zero."""
    return np.trunc(timesteps(n_steps, shift, s_max)).astype(np.int64)
