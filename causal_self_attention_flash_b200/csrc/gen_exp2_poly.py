"""Minimax polynomial for 2^f on [-1/2, 1/2] by the Remez exchange algorithm.

    python gen_exp2_poly.py [degree]

The kernels evaluate part of their exponentials as 2^x = 2^j * p(x - j) with
j = round(x), on the FMA pipes, next to the hardware ex2 unit.  This script
computes the coefficients of p (minimising the maximum *relative* error
|p(f) / 2^f - 1|, the quantity that matters for the softmax sums), prints
them as C++ float literals, and reports the error bound achieved in exact
arithmetic and after rounding the coefficients to float32.

Method: Remez exchange (E. Remez, 1934) on the weighted error
e(f) = (p(f) - 2^f) / 2^f, starting from Chebyshev extrema; each step solves
the linear system p(x_i) - 2^x_i = (-1)^i E 2^x_i at n+2 reference points
and moves the references to the extrema of e.
"""

from __future__ import annotations

import sys

import numpy as np

A, B = -0.5, 0.5


def remez(degree: int, iters: int = 30):
    n = degree
    k = np.arange(n + 2)
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * (n + 1 - k) / (n + 1))
    grid = np.linspace(A, B, 200001)
    coef = None
    for _ in range(iters):
        f = np.exp2(x)
        M = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            M[i, : n + 1] = x[i] ** np.arange(n + 1)
            M[i, n + 1] = (-1) ** i * f[i]
        sol = np.linalg.solve(M, f)
        coef = sol[: n + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # new references: alternating extrema of err
        sign = np.sign(err)
        idx = [0]
        for i in range(1, len(grid)):
            if sign[i] != sign[idx[-1]]:
                idx.append(i)
            elif abs(err[i]) > abs(err[idx[-1]]):
                idx[-1] = i
        if len(idx) >= n + 2:
            best = max(range(len(idx) - n - 1),
                       key=lambda s: min(abs(err[j]) for j in idx[s:s + n + 2]))
            x = grid[idx[best:best + n + 2]]
    return coef


def max_rel_err(coef, as_f32: bool):
    g = np.linspace(A, B, 400001)
    if as_f32:
        c = np.asarray(coef, dtype=np.float32).astype(np.float64)
    else:
        c = np.asarray(coef, dtype=np.float64)
    p = np.polyval(c[::-1], g)
    return float(np.max(np.abs(p / np.exp2(g) - 1.0)))


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 5
    coef = remez(degree)
    print(f"// degree {degree}, minimax relative error on [-1/2, 1/2]: "
          f"{max_rel_err(coef, False):.3e} (float32 coefficients: "
          f"{max_rel_err(coef, True):.3e})")
    for i, c in enumerate(coef):
        print(f"constexpr float kExp2C{i} = {float(np.float32(c))!r}f;")


if __name__ == "__main__":
    main()
