"""Coefficients of the FMA-pipe exp2 used by the prefill softmax.

2^x is evaluated as 2^n * p(f) with n = floor(x), f = x - n in [0, 1)
(argument reduction in the manner of Cody and Waite, base 2), where p is the
polynomial of the given degree that minimises the maximum RELATIVE error
|p(f) / 2^f - 1| on [0, 1], found with the Remez exchange algorithm.  The
probabilities this feeds are rounded to bf16 (relative step 2^-8), so degree 3
(max relative error about 9e-5) is ample.

    python gen_exp2_poly.py [degree]

prints the coefficients c0..c_deg (p(f) = c0 + c1 f + ... ) and the error.
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 60):
    n = deg + 2
    # initial reference: Chebyshev extrema on [0, 1]
    x = 0.5 - 0.5 * np.cos(np.pi * np.arange(n) / (n - 1))
    grid = np.linspace(0.0, 1.0, 200001)
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative equioscillation)
        A = np.zeros((n, n))
        for i, xi in enumerate(x):
            A[i, :deg + 1] = xi ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** xi
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extrema of the error between sign changes
        sign_change = np.nonzero(np.diff(np.sign(err)))[0]
        bounds = np.concatenate([[0], sign_change + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(deg)
    for k, v in enumerate(c):
        print(f"c{k} = {v:.9e}f")
    print(f"max relative error = {e:.3e}")
