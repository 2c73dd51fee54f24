"""Remez exchange for the cubic behind the FMA-pipe 2^x of the attention
softmax (``ex2_poly2`` in the kernels' PTX helper header).

The kernel computes 2^x as 2^n * p(f) with n = rint(x) and f = x - n in
[-1/2, 1/2] (Cody-Waite range reduction: the integer part goes into the
exponent field).  p is the cubic c0 + c1 f + c2 f^2 + c3 f^3 that minimises
the largest RELATIVE error max |p(f) / 2^f - 1| on [-1/2, 1/2].  By the
equioscillation theorem the best such cubic makes the weighted error reach
its maximum E with alternating signs at 5 points; the Remez exchange finds
them: solve p(x_i) - 2^{x_i} = (-1)^i E 2^{x_i} on the current 5 points,
move each point to the extremum of the error on its sign run, repeat.

    python tests/golden/ex2_cubic_fit.py      # prints c3, c2, c1, c0 and E

Plain float64 numpy: this is a fit of a function from mathematics; it uses
nothing of CUDA's math library.
"""
from __future__ import annotations

import numpy as np


def remez_relative(deg: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 40, grid: int = 200001):
    """Coefficients c0..c_deg (ascending) of the minimax-relative-error
    polynomial for 2^f on [a, b], and the levelled error E."""
    n = deg + 2
    k = np.arange(n)
    x = (a + b) / 2 - (b - a) / 2 * np.cos(np.pi * k / (n - 1))  # Chebyshev extrema as the first reference
    g = np.linspace(a, b, grid)
    E = 0.0
    for _ in range(iters):
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = (-1.0) ** k * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c, E = sol[:deg + 1], abs(sol[deg + 1])
        err = np.polyval(c[::-1], g) / np.exp2(g) - 1.0
        # one extremum per run of constant sign
        runs = np.flatnonzero(np.diff(np.sign(err)) != 0) + 1
        bounds = np.concatenate([[0], runs, [len(g)]])
        idx = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(idx) != n:
            raise RuntimeError(f"expected {n} alternations, found {len(idx)}")
        x_new = g[idx]
        if np.allclose(x_new, x, rtol=0, atol=1e-12):
            break
        x = x_new
    return c, E


def max_relative_error(c_ascending, a: float = -0.5, b: float = 0.5, grid: int = 400001) -> float:
    g = np.linspace(a, b, grid)
    return float(np.max(np.abs(np.polyval(np.asarray(c_ascending)[::-1], g) / np.exp2(g) - 1.0)))


if __name__ == "__main__":
    c, E = remez_relative()
    print("c3 = %.11f\nc2 = %.11f\nc1 = %.11f\nc0 = %.11f\nE  = %.3e" % (c[3], c[2], c[1], c[0], E))
