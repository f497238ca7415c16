"""The FMA-pipe base-2 exponential of the attention softmax: the fp32
evaluation sequence (same operations, same order as the kernel) checked
against numpy's float64 exp2, and the kernel's constants checked against
the committed fit."""

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "video_diffusion_transformer_self_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location(
        "fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "attention.cu")).read()
    body = src[src.index("exp2_fma2(float2 x)"):]
    body = body[:body.index("\n}\n")]
    vals = re.findall(r"make_float2\(([-0-9.e+]+)f, \1f\)", body)
    # magic, c3, c2, c1, c0 in the order they appear
    return [float(v) for v in vals]


def test_polynomial_accuracy():
    fit = _fit_module()
    c = [float(np.float32(v)) for v in fit.fit()]
    x = np.linspace(-126.0, 8.0, 400001)
    y = fit.eval_fp32(x, c).astype(np.float64)
    rel = np.abs(y / np.exp2(x) - 1.0)
    assert rel.max() < 2e-4
    # exact at integers (p(0) = 1, exponent added exactly)
    xi = np.arange(-126, 9, dtype=np.float64)
    assert np.array_equal(fit.eval_fp32(xi, c).astype(np.float64),
                          np.exp2(xi))
    # clamped below: never wraps to a large value
    yl = fit.eval_fp32(np.array([-200.0, -1e30, -127.5]), c)
    assert np.all(yl >= 0) and np.all(yl <= 2.0 ** -125)


def test_kernel_uses_the_fitted_constants():
    fit = _fit_module()
    want = [float(np.float32(v)) for v in fit.fit()]  # c0, c1, c2, c3
    got = _kernel_coefficients()
    assert got[0] == 12582912.0
    c3, c2, c1, c0 = got[1:5]
    for g, w in zip((c0, c1, c2, c3), want):
        assert abs(g - w) <= 1e-9 * max(1.0, abs(w)), (g, w)
