"""Derivation of the polynomial exp2 used on the FMA pipe by the attention kernel.

2^x is split as x = r + f with r = round(x) (an integer, added to the float's
exponent field) and f in [-1/2, 1/2].  2^f is approximated by a degree-3
polynomial whose coefficients minimise the maximum relative error on
[-1/2, 1/2]: a Remez exchange on the relative error, started from a
least-squares fit at Chebyshev nodes.  The float32-rounded coefficients reach
a maximum relative error of about 7.5e-5, far below the 2^-9 relative
rounding of the bf16 probabilities they feed.

Run it to print the coefficients; csrc/sm100.cuh holds them as float literals.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3


def fit(degree: int = DEGREE, iters: int = 30):
    grid = np.linspace(-0.5, 0.5, 200001)
    nodes = 0.5 * np.cos(np.pi * (np.arange(200) + 0.5) / 200)
    A = np.vander(nodes, degree + 1, increasing=True) / (2.0 ** nodes)[:, None]
    c, *_ = np.linalg.lstsq(A, np.ones_like(nodes), rcond=None)
    for _ in range(iters):
        err = (np.polyval(c[::-1], grid) - 2 ** grid) / 2 ** grid
        ext = np.r_[0, np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1, len(grid) - 1]
        ext = np.sort(ext[np.argsort(-np.abs(err[ext]))][: degree + 2])
        x = grid[ext]
        M = np.hstack([np.vander(x, degree + 1, increasing=True) / (2.0 ** x)[:, None],
                       ((-1.0) ** np.arange(degree + 2))[:, None]])
        c = np.linalg.solve(M, np.ones(degree + 2))[: degree + 1]
    c32 = c.astype(np.float32)
    err = (np.polyval(c32[::-1].astype(np.float64), grid) - 2 ** grid) / 2 ** grid
    return c32, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = fit()
    print("coefficients c0..c3:", ", ".join(f"{float(v):.9g}f" for v in c), f"max rel err {e:.3g}")
