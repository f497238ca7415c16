"""Host side of the UniPC step (no GPU): the library's folded coefficients
equal the ones read off the oracle's corrector and predictor (both are
linear in their inputs, so unit inputs give the coefficients), and bad
schedules, indices and pointers are rejected before any device call."""

import ctypes
import math

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as hst

from oracle import schedule, unipc
from video_diffusion_transformer_self_b200 import build, wan


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wan.lib()


def oracle_coeffs(sig, i):
    """Coefficients of the oracle's steps, probed with unit inputs."""
    def corr(xc, m2, m1, m):
        md = {i: np.array([m]), i - 1: np.array([m1])}
        if i >= 2:
            md[i - 2] = np.array([m2])
        return float(unipc.corrector(np.array([xc]), md, sig, i)[0])

    def pred(xc, m1, m):
        md = {i: np.array([m])}
        if i >= 1:
            md[i - 1] = np.array([m1])
        return float(unipc.predictor(np.array([xc]), md, sig, i)[0])

    c = {"px": pred(1, 0, 0), "pm1": pred(0, 1, 0), "pm": pred(0, 0, 1)}
    if i >= 1:
        c.update(cx=corr(1, 0, 0, 0), cm2=corr(0, 1, 0, 0),
                 cm1=corr(0, 0, 1, 0), cm=corr(0, 0, 0, 1))
    else:
        c.update(cx=0.0, cm2=0.0, cm1=0.0, cm=0.0)
    return c


SCHEDULES = [(40, 12.0, 1.0), (40, 12.0, 0.999), (40, 5.0, 1.0),
             (10, 3.0, 0.9), (3, 1.0, 1.0), (1, 12.0, 1.0)]


@pytest.mark.parametrize("n,shift,smax", SCHEDULES)
def test_coefficients_match_oracle(lib, n, shift, smax):
    sig = schedule.sigmas(n, shift, smax)
    for i in range(n):
        got = wan.unipc_coeffs(sig, i)
        want = oracle_coeffs(sig, i)
        assert got["sigma"] == sig[i]
        for key, w in want.items():
            assert got[key] == pytest.approx(w, rel=1e-11, abs=1e-14), \
                (i, key, got[key], w)
        assert got["pred_order"] == unipc.predictor_order(sig, i)
        if i == 0:
            assert got["corr_order"] == 0
        else:
            assert got["corr_order"] == unipc.predictor_order(sig, i - 1)


def test_coefficients_structure(lib):
    sig = schedule.sigmas(40, 12.0)
    c0 = wan.unipc_coeffs(sig, 0)
    # first stop: the Euler step (px x + pm (x - sigma v) = x + dsigma v)
    assert c0["px"] + c0["pm"] == pytest.approx(1.0, abs=1e-15)
    assert c0["pm"] * sig[0] == pytest.approx(sig[0] - sig[1], rel=1e-13)
    last = wan.unipc_coeffs(sig, 39)
    assert (last["px"], last["pm"], last["pm1"]) == (0.0, 1.0, 0.0)
    for i in range(40):
        c = wan.unipc_coeffs(sig, i)
        # constant data prediction is kept exactly: m -> m
        assert c["px"] + c["pm"] + c["pm1"] == pytest.approx(1.0, abs=1e-13)
        if i:
            assert c["cx"] + c["cm1"] + c["cm2"] + c["cm"] == \
                pytest.approx(1.0, abs=1e-13)


def test_rejects(lib):
    L = lib
    out = wan.UniPCCoef()
    good = schedule.sigmas(4, 5.0)
    arr = (ctypes.c_double * 5)(*good)
    assert L.wan_unipc_coeffs(arr, 4, 4, ctypes.byref(out)) == wan.WAN_EINVAL
    assert L.wan_unipc_coeffs(arr, 4, -1, ctypes.byref(out)) == wan.WAN_EINVAL
    assert L.wan_unipc_coeffs(arr, 0, 0, ctypes.byref(out)) == wan.WAN_EINVAL
    assert L.wan_unipc_coeffs(None, 4, 0, ctypes.byref(out)) == wan.WAN_EINVAL
    for bad in ([1.0, 0.5, 0.5, 0.2, 0.0], [1.2, 0.5, 0.3, 0.2, 0.0],
                [1.0, 0.5, 0.3, 0.0, 0.0], [1.0, math.nan, 0.3, 0.2, 0.0],
                [1.0, 0.5, 0.3, 0.2, -0.1]):
        b = (ctypes.c_double * 5)(*bad)
        assert L.wan_unipc_coeffs(b, 4, 0, ctypes.byref(out)) == \
            wan.WAN_EINVAL, bad
    p = ctypes.c_void_p
    x, xc, m1, m2, mo, vc = (p(4096 * k) for k in range(1, 7))
    st = L.wan_unipc_step
    # aliasing: x_corr == x; m_out == m_prev1; m_out == v_cond
    assert st(x, x, m1, m2, mo, vc, None, 1.0, 8, arr, 4, 2, None) \
        == wan.WAN_EINVAL
    assert st(x, xc, m1, m2, m1, vc, None, 1.0, 8, arr, 4, 2, None) \
        == wan.WAN_EINVAL
    assert st(x, xc, m1, m2, vc, vc, None, 1.0, 8, arr, 4, 2, None) \
        == wan.WAN_EINVAL
    # m_prev1 required from stop 1 on, m_prev2 once the corrector is order 2
    assert st(x, xc, None, m2, mo, vc, None, 1.0, 8, arr, 4, 1, None) \
        == wan.WAN_EINVAL
    sig40 = (ctypes.c_double * 41)(*schedule.sigmas(40, 12.0))
    assert st(x, xc, m1, None, mo, vc, None, 1.0, 8, sig40, 40, 20, None) \
        == wan.WAN_EINVAL
    assert st(p(4100), xc, m1, m2, mo, vc, None, 1.0, 8, arr, 4, 2, None) \
        == wan.WAN_EALIGN
    assert st(x, xc, m1, m2, mo, vc, None, math.inf, 8, arr, 4, 2, None) \
        == wan.WAN_EINVAL
    assert st(None, None, None, None, None, None, None, 1.0, 0, arr, 4, 2,
              None) == wan.WAN_OK  # empty: nothing to do


@hst.composite
def schedules(draw):
    n = draw(hst.integers(1, 30))
    shift = draw(hst.floats(0.5, 20.0))
    smax = draw(hst.sampled_from([1.0, 0.999, 0.95, 0.7]))
    return schedule.sigmas(n, shift, smax)


@settings(max_examples=40, deadline=None)
@given(schedules(), hst.data())
def test_coefficients_match_oracle_random_schedules(sig, data):
    build.build()
    n = len(sig) - 1
    i = data.draw(hst.integers(0, n - 1))
    got = wan.unipc_coeffs(sig, i)
    want = oracle_coeffs(sig, i)
    for key, w in want.items():
        assert got[key] == pytest.approx(w, rel=1e-10, abs=1e-13), (key, i)
