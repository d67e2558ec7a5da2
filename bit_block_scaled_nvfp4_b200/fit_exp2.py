"""Fit of the polynomial p(f) ~ 2^f on [-1/2, 1/2] used by the prefill kernel's exp2 on the FMA
pipe (2^t = 2^n p(t - n), n = round(t)).

Weighted least squares on Chebyshev nodes, reweighted towards the minimax (relative) error
(Lawson's iteration). Run as a script to print the coefficients (rounded to fp32) and the
maximum relative error of the fp32 coefficients in exact arithmetic.
"""
import numpy as np


def fit(degree: int = 5, nodes: int = 4000, iters: int = 200):
    f = 0.5 * np.cos(np.pi * (np.arange(nodes) + 0.5) / nodes)
    y = 2.0 ** f
    a = np.vstack([f ** k for k in range(degree + 1)]).T
    w = np.ones(nodes)
    for _ in range(iters):
        sw = np.sqrt(w) / y
        c, *_ = np.linalg.lstsq(a * sw[:, None], y * sw, rcond=None)
        e = (a @ c - y) / y
        w = w * np.sqrt(np.abs(e)) + 1e-300
        w /= w.sum()
    c32 = c.astype(np.float32).astype(np.float64)
    ff = np.linspace(-0.5, 0.5, 400001)
    err = np.max(np.abs(np.polyval(c32[::-1], ff) / 2.0 ** ff - 1.0))
    return c.astype(np.float32), err


if __name__ == "__main__":
    c, err = fit()
    for k, v in enumerate(c):
        print(f"c{k} = {float(v)!r}f")
    print(f"max relative error {err:.3e}")
