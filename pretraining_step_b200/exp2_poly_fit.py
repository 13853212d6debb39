"""Coefficients of the polynomial 2^f on [-1/2, 1/2] that the attention
kernels evaluate on the FMA pipe for part of their softmax exponentials.

Method: the Remez exchange algorithm for the best approximation in the
minimax sense, here of the RELATIVE error (p(f) - 2^f) / 2^f, since the
result is scaled by 2^n afterwards and then rounded to bf16.  Starting from
Chebyshev extrema, each pass solves the linear system
    p(x_i) - 2^x_i = (-1)^i E 2^x_i,   i = 0 .. degree + 1
for the coefficients and the levelled error E, then moves the reference
points to the extrema of the new error curve, until they stop moving.

Run as a script it prints the coefficients (degree 3 by default) as the C
literals of csrc/exp2_poly.cuh and the maximum relative error.
"""
import sys

import numpy as np


def fit(degree=3, passes=40, grid=400001):
    """Minimax (relative error) polynomial for 2^f on [-1/2, 1/2].

    Returns (coefficients c_0 .. c_degree, lowest power first; max |relative
    error| of the fp64 polynomial on a dense grid)."""
    n = degree + 2
    x = 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))[::-1]
    g = np.linspace(-0.5, 0.5, grid)
    c = None
    for _ in range(passes):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1.0) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = rel_error(c, g)
        # One extremum per run of constant sign: the new reference.
        ext, start = [], 0
        sign = np.sign(err)
        for j in range(1, grid):
            if sign[j] != sign[j - 1]:
                ext.append(start + int(np.argmax(np.abs(err[start:j]))))
                start = j
        ext.append(start + int(np.argmax(np.abs(err[start:]))))
        if len(ext) != n:
            break
        nx = g[ext]
        if np.max(np.abs(nx - x)) < 1e-12:
            break
        x = nx
    return c, float(np.max(np.abs(rel_error(c, g))))


def rel_error(c, f):
    """(p(f) - 2^f) / 2^f in fp64 for coefficients c (lowest power first)."""
    p = np.zeros_like(f)
    for ck in c[::-1]:
        p = p * f + ck
    return (p - 2.0 ** f) / 2.0 ** f


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = fit(deg)
    for k, ck in enumerate(c):
        print(f"c{k} = {float(np.float32(ck))!r}f")
    print(f"max relative error {e:.3e}")
