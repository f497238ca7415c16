"""Fit the polynomial of the FMA-pipe base-2 exponential used in the
attention softmax (attention.cu, ``exp2_fma``).

Method (Cody-Waite style range reduction, polynomial fitted here):
  x = n + f with n = round-to-nearest(x) (the 1.5 * 2^23 add trick, so n
  sits in the low mantissa bits) and f in [-0.5, 0.5];
  2^x = 2^n * p(f), p a degree-3 polynomial fitted by weighted least
  squares to 2^f on Chebyshev nodes of [-0.5, 0.5], minimising the
  relative error, with p(0) pinned to 1 so 2^n is exact at integers;
  2^n is applied by adding n << 23 to the bit pattern of p(f).

Run:  python fit_exp2.py      prints the coefficients and the max relative
error of the fp32 evaluation (Horner, fused multiply-adds) over a dense
grid, measured against numpy's float64 exp2.
"""

import numpy as np


def fit(degree=3, nodes=4096):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)  # Chebyshev nodes
    y = np.exp2(f)
    # p(f) = 1 + c1 f + c2 f^2 + c3 f^3, relative error weighting 1 / y
    A = np.stack([f ** i for i in range(1, degree + 1)], axis=1) / y[:, None]
    b = (y - 1.0) / y
    c, *_ = np.linalg.lstsq(A, b, rcond=None)
    return np.concatenate([[1.0], c])


def eval_fp32(x, c):
    """Evaluate exactly as the kernel does, in float32."""
    x = np.asarray(x, np.float32)
    x = np.maximum(x, np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    j = (x + magic).astype(np.float32)
    n = (j - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    c = [np.float32(v) for v in c]
    p = c[3]
    for ci in (c[2], c[1], c[0]):
        # fused multiply-add: one rounding
        p = (p.astype(np.float64) * f.astype(np.float64)
             + np.float64(ci)).astype(np.float32)
    bits = p.view(np.int32) + (j.view(np.int32) - np.int32(0x4B400000)) * \
        np.int32(1 << 23)
    return bits.astype(np.int32).view(np.float32)


if __name__ == "__main__":
    c = fit()
    c32 = [float(np.float32(v)) for v in c]
    x = np.linspace(-126.0, 8.0, 2000001)
    y = eval_fp32(x, c32).astype(np.float64)
    rel = np.abs(y / np.exp2(x) - 1.0)
    print("coefficients (fp32):", ", ".join("%.9ef" % v for v in c32))
    print("max relative error on [-126, 8]: %.3e" % rel.max())
