"""Fits the polynomial p(f) ~ 2^f on [-1/2, 1/2] that the attention kernel uses
to evaluate part of its exponentials on the FMA pipe instead of the MUFU unit.

Evaluation in the kernel: x = n + f with n = round-to-nearest(x) (obtained by
adding 1.5 * 2^23 in fp32), f = x - n, then 2^x = 2^n * p(f), the 2^n factor
applied by adding n to the exponent field of p(f).

Fit: weighted least squares on Chebyshev nodes of [-1/2, 1/2] with weights
2^-f, so the error minimised is the relative one; p(0) = 1 is imposed exactly.
The coefficients are rounded to fp32 and the relative error of the fp32 Horner
evaluation is measured on a dense grid.

    python -m sparse_attention_hyb_b200.fit_exp2_poly [degree]
"""
import sys

import numpy as np


def fit(deg: int, n_nodes: int = 4096):
    k = np.arange(n_nodes)
    f = -0.5 * np.cos(np.pi * (k + 0.5) / n_nodes)              # Chebyshev nodes on [-1/2, 1/2]
    y = np.exp2(f)
    w = 1.0 / y
    A = np.stack([f ** i for i in range(1, deg + 1)], axis=1) * w[:, None]
    c, *_ = np.linalg.lstsq(A, (y - 1.0) * w, rcond=None)
    coef = np.concatenate([[1.0], c]).astype(np.float32)
    g = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    acc = np.full_like(g, coef[-1])
    for ci in coef[-2::-1]:
        acc = (acc * g + ci).astype(np.float32)
    rel = np.abs(acc.astype(np.float64) / np.exp2(g.astype(np.float64)) - 1.0)
    return coef, float(rel.max())


if __name__ == "__main__":
    d = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    coef, err = fit(d)
    print("coefficients (f^0 .. f^%d):" % d, [float(x) for x in coef], [float(x).hex() for x in coef])
    print("max relative error of fp32 Horner evaluation on [-1/2, 1/2]: %.3e" % err)
