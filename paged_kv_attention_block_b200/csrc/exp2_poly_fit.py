"""Fit of the cubic used by exp2_fma2 (common.cuh): 2^f on [-1/2, 1/2].

Weighted least squares on Chebyshev nodes, minimising the relative error, with
the weights moved towards the error's extrema at every round (Lawson's
iteration), which approaches the equal-ripple (minimax) fit.  Prints the four
coefficients rounded to float32 and the largest relative error of the float32
evaluation (Horner's scheme), which common.cuh states.

    python exp2_poly_fit.py
"""
import numpy as np


def fit(degree: int = 3, nodes: int = 4000, rounds: int = 200):
    k = np.arange(nodes)
    f = 0.5 * np.cos(np.pi * (k + 0.5) / nodes)
    y = 2.0 ** f
    A = np.vstack([f ** i for i in range(degree + 1)]).T / y[:, None]
    w = np.ones(nodes)
    for _ in range(rounds):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(A * sw[:, None], sw, rcond=None)
        e = np.abs(A @ c - 1.0)
        w = w * (e + 1e-18)
        w /= w.sum()
    return [np.float32(x) for x in c]


def max_rel_error(c32) -> float:
    f = np.linspace(-0.5, 0.5, 200001).astype(np.float32)
    p = np.float32(0)
    for coef in reversed(c32):
        p = p * f + coef
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c = fit()
    print("coefficients (c0..c3):", ", ".join(f"{float(x):.8g}f" for x in c))
    print("max relative error:", max_rel_error(c))
