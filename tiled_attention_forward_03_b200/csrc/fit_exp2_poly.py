"""Fit the polynomial the kernel uses for 2^f on f in [-1/2, 1/2].

The kernel evaluates part of its exponentials 2^x on the FMA pipe instead of the
special-function unit: x = n + f with n = round(x) and |f| <= 1/2, 2^x = 2^n * p(f),
where 2^n is applied by adding n to the float's exponent field (Cody-Waite style
range reduction with a single step, exact because n is an integer and f = x - n is
computed exactly in fp32 for |x| < 2^22).

p is the degree-d polynomial minimising the maximum RELATIVE error |p(f)/2^f - 1|
over [-1/2, 1/2], found here with the Remez exchange algorithm (linear system on
d+2 alternation points, then moving the points to the extrema of the error, until
the levelled error stops changing).  The coefficients are then rounded to fp32 and
the error is re-measured on a dense grid with fp32 Horner evaluation.

    python fit_exp2_poly.py [degree]
"""
from __future__ import annotations

import sys

import numpy as np


def remez_relative(deg: int, a: float = -0.5, b: float = 0.5, iters: int = 40):
    f = lambda t: np.exp2(t)
    k = np.arange(deg + 2)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (deg + 1 - k) / (deg + 1))  # Chebyshev extrema
    grid = np.linspace(a, b, 200001)
    E = 0.0
    for _ in range(iters):
        # p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error levelled at the reference)
        A = np.zeros((deg + 2, deg + 2))
        for i, xi in enumerate(x):
            A[i, : deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(xi)
        sol = np.linalg.solve(A, f(x))
        c, E = sol[: deg + 1], sol[deg + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        # new reference: the extremum of err on each sign-constant run
        s = np.sign(err)
        s[s == 0] = 1
        runs = np.split(np.arange(grid.size), np.where(np.diff(s) != 0)[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < deg + 2:
            break
        # keep deg+2 consecutive extrema with the largest minimum magnitude
        best = max(range(len(ext) - deg - 1), key=lambda i: np.min(np.abs(err[ext[i:i + deg + 2]])))
        x_new = grid[ext[best: best + deg + 2]]
        if np.allclose(x_new, x, atol=1e-12):
            break
        x = x_new
    return c, abs(E)


def fp32_horner_error(c32: np.ndarray, a: float = -0.5, b: float = 0.5) -> float:
    t = np.linspace(a, b, 400001).astype(np.float32)
    p = np.full_like(t, c32[-1])
    for ci in c32[-2::-1]:
        p = (p * t + ci).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(t.astype(np.float64)) - 1.0)))


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, E = remez_relative(deg)
    c32 = c.astype(np.float32)
    print(f"degree {deg}: levelled relative error {E:.3e}; fp32 Horner max relative error "
          f"{fp32_horner_error(c32):.3e}")
    for i, ci in enumerate(c32):
        print(f"  c{i} = {float(ci)!r}f  ({ci.view(np.uint32):#010x})")


if __name__ == "__main__":
    main()
