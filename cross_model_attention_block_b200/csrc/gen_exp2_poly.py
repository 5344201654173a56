"""Coefficients of the FMA-pipe exp2 used by the block-statistics kernel.

    python cross_model_attention_block_b200/csrc/gen_exp2_poly.py [degree]

2^x is split as 2^j * 2^f with j = round(x) and f in [-1/2, 1/2]; 2^f is
approximated by a polynomial p(f) = c0 + c1 f + ... + cn f^n chosen to
minimise the largest relative error max |p(f) / 2^f - 1| over the interval
(minimax in the relative sense).  The fit is a Remez exchange: start from
Chebyshev extrema, solve for the polynomial that equioscillates on the
reference set, move the reference to the extrema of the new error curve, and
repeat until the levelled error stops changing.  Everything runs in float64;
the printed float32 constants are then re-scored with float32 Horner
evaluation so the table in tc_qk.cu carries its real error.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(degree: int, iters: int = 30):
    a, b = -0.5, 0.5
    n = degree + 2  # reference points
    k = np.arange(n)
    ref = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(a, b, 200001)
    level = None
    for _ in range(iters):
        # p(x_i) - 2^x_i * (-1)^i * E = 2^x_i  (relative error levelled at E)
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1.0) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        c, level = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum per sign-alternating run of the error
        sgn = np.sign(err)
        cuts = np.flatnonzero(np.diff(sgn) != 0) + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs if r.size]
        if len(ext) < n:
            break
        ext = np.array(ext)
        while ext.size > n:  # drop the smallest end extremum
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        ref = grid[ext]
    return c, abs(level)


def float32_error(c32: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = np.full_like(f, c32[-1])
    for ck in c32[-2::-1]:
        p = (p * f + ck).astype(np.float32)
    return float(np.max(np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)))


def main():
    degree = int(sys.argv[1]) if len(sys.argv) > 1 else 4
    c, e = remez_exp2(degree)
    c32 = c.astype(np.float32)
    print(f"// degree {degree}: levelled relative error {e:.3e} (float64), "
          f"{float32_error(c32):.3e} with float32 coefficients and Horner steps")
    for i, ci in enumerate(c32):
        print(f"constexpr float kExp2C{i} = {float(ci)!r}f;")


if __name__ == "__main__":
    main()
