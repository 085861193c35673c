"""Fits the polynomial that the prefill kernel uses for part of its exp2.

The kernel evaluates 2^x as 2^j * p(f) with j = round(x), f = x - j in
[-1/2, 1/2] (Cody-Waite style range reduction; the scaling by 2^j is an
integer add into the exponent field). p is a degree-3 polynomial fitted
here, constant term 1, by weighted least squares on Chebyshev nodes, refined with Lawson
iterations (iteratively reweighted least squares) toward the minimax
relative error. Run ``python -m sink_augmented_gqa_b200.fit_exp2_poly`` to
reproduce the coefficients in ``csrc/ptx.cuh``; ``tests/test_exp2_poly.py``
checks that the two agree and that the fp32 Horner evaluation keeps the
relative error below 1.5e-4 (bf16 P carries 2^-9).
"""

import numpy as np

DEGREE = 3


def fit(degree=DEGREE, nodes=4000, iters=60):
    """p(f) = 1 + c1 f + ... + c_degree f^degree with the constant term pinned
    to 1, so that 2^x comes out exact at integer x (x = 0 gives exactly 1)."""
    f = np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes) * 0.5
    y = np.exp2(f)
    w = np.ones_like(f)
    c = None
    for _ in range(iters):
        # relative error (1 + sum_k c_k f^k) / y - 1, linear in c_1..c_degree
        A = np.vander(f, degree + 1, increasing=True)[:, 1:] / y[:, None]
        rhs = 1.0 - 1.0 / y
        c, *_ = np.linalg.lstsq(A * np.sqrt(w)[:, None], rhs * np.sqrt(w), rcond=None)
        err = np.abs((1.0 + np.polyval(np.r_[c[::-1], 0.0], f)) / y - 1)
        w = w * (err + 1e-30)
        w /= w.sum()
    return np.r_[1.0, c].astype(np.float32)


def horner_fp32(c, f):
    f = np.asarray(f, dtype=np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    return p


def max_rel_error(c, n=200001):
    f = np.linspace(-0.5, 0.5, n).astype(np.float32)
    return float(np.abs(horner_fp32(c, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1).max())


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", ", ".join(f"{float(x):.9g}f" for x in c))
    print("max relative error:", max_rel_error(c))
