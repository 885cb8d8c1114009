"""Fits the degree-3 polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the fused
forward kernel to evaluate part of its softmax exponentials on the FMA pipe
(Cody-Waite range reduction 2^x = 2^round(x) * 2^(x - round(x))).

Method: minimax in relative error by iteratively reweighted least squares on
Chebyshev nodes (Lawson's algorithm). Prints the fp32 coefficients c0..c3 and
the maximum relative error of fp32 Horner evaluation.

    python block_sparse_attention_cov_b200/csrc/fit_exp2_poly.py
"""
import numpy as np


def fit(deg=3, iters=200):
    f = np.cos(np.linspace(0.0, np.pi, 4001)) * 0.5
    y = 2.0 ** f
    w = np.ones_like(f)
    V = np.vander(f, deg + 1, increasing=True)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq((V / y[:, None]) * w[:, None], w, rcond=None)
        err = (V @ c - y) / y
        w = w * (1.0 + 0.5 * np.abs(err) / np.abs(err).max())
    return c.astype(np.float32)


def horner32(c, f):
    f = np.asarray(f, np.float32)
    p = np.float32(c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + np.float32(c[k])).astype(np.float32)
    return p


if __name__ == "__main__":
    c = fit()
    ff = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    rel = np.abs(horner32(c, ff).astype(np.float64) - 2.0 ** ff.astype(np.float64)) / 2.0 ** ff.astype(np.float64)
    for i, x in enumerate(c):
        print(f"c{i} = {float(x)!r}f")
    print("max relative error", rel.max())
