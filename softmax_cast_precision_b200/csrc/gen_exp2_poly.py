"""Generate the polynomial that the kernels use for 2^f on [-1/2, 1/2].

Method (range reduction in the style of Cody and Waite, then a minimax
polynomial fitted here): 2^x = 2^j * 2^f with j = round(x) and
f = x - j in [-1/2, 1/2]; 2^f is approximated by a degree-4 polynomial whose
coefficients minimise the maximum relative error on that interval, found by
the Remez exchange algorithm in float64 and then rounded to float32.

    python gen_exp2_poly.py          # prints the coefficients and their error

The printed constants are pasted into sm100_ptx.cuh (exp2_poly_*); the
test suite re-runs this fit and checks that they agree.
"""
from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def _solve(nodes: np.ndarray) -> tuple[np.ndarray, float]:
    """Coefficients c and levelled error E with (p(x_i) - 2^x_i) / 2^x_i = (-1)^i E."""
    n = DEGREE + 2
    A = np.zeros((n, n))
    for i, x in enumerate(nodes):
        A[i, :DEGREE + 1] = x ** np.arange(DEGREE + 1) / 2.0 ** x
        A[i, DEGREE + 1] = -((-1.0) ** i)
    sol = np.linalg.solve(A, np.ones(n))
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def rel_error(c: np.ndarray, x: np.ndarray) -> np.ndarray:
    return np.polynomial.polynomial.polyval(x, c) / 2.0 ** x - 1.0


def remez(iters: int = 30) -> np.ndarray:
    k = np.arange(DEGREE + 2)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (DEGREE + 1))  # Chebyshev extrema
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(nodes)
        err = rel_error(c, grid)
        # new nodes: the alternating extrema of the error curve
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) < DEGREE + 2:
            break
        # keep the DEGREE + 2 largest alternating extrema
        while len(ext) > DEGREE + 2:
            drop = int(np.argmin([abs(err[e]) for e in (ext[0], ext[-1])]))
            ext = ext[1:] if drop == 0 else ext[:-1]
        nodes = grid[ext]
    return c


def coefficients_f32() -> np.ndarray:
    return remez().astype(np.float32)


def max_rel_error_f32(c32: np.ndarray) -> float:
    """Worst relative error of the float32 Horner evaluation on the interval."""
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ci in c32[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0)))


if __name__ == "__main__":
    c = coefficients_f32()
    for i, ci in enumerate(c):
        print(f"c{i} = {float(ci).hex()}  ({ci:.9e})")
    print("max relative error (float32 Horner):", max_rel_error_f32(c))
