"""Fit the polynomial the attention kernel uses for part of its base-2
exponentials.

    python full_gqa_learned_b200/csrc/exp2_poly_fit.py

2^x is split as 2^n * 2^f with n = round-to-nearest(x) and f in [-1/2, 1/2]
(Cody and Waite's additive range reduction).  2^f is approximated by a degree
4 polynomial whose coefficients minimise the maximum relative error on
[-1/2, 1/2]: a least-squares start on Chebyshev nodes refined by Lawson's
iteratively reweighted least squares, which converges to the minimax
(equioscillating) solution.  Prints the coefficients as C++ float literals
and the relative error they reach.
"""
import numpy as np

DEG = 4


def fit(deg=DEG, iters=200):
    f = np.cos(np.pi * (np.arange(4001) + 0.5) / 4001) * 0.5      # Chebyshev nodes
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True) / y[:, None]       # relative error system
    w = np.ones_like(f) / f.size
    for _ in range(iters):
        sw = np.sqrt(w)
        c, *_ = np.linalg.lstsq(V * sw[:, None], sw, rcond=None)
        e = np.abs(V @ c - 1.0)
        w = w * (e + 1e-300)
        w /= w.sum()
    return c


def rel_error(c32):
    x = np.linspace(-0.5, 0.5, 200001)
    p = np.zeros_like(x, dtype=np.float64)
    for k in reversed(range(len(c32))):
        p = p * x + np.float64(c32[k])
    return float(np.max(np.abs(p / np.exp2(x) - 1.0)))


if __name__ == "__main__":
    c = fit()
    c32 = c.astype(np.float32)
    for k, v in enumerate(c32):
        print("constexpr float kExp2C%d = %.9ef;" % (k, v))
    print("// max relative error on [-1/2, 1/2]: %.3e" % rel_error(c32))
