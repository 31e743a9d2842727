"""Coefficients of the polynomial behind the FMA-pipe exp2 in fwd_bf16.cu.

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2] (Cody and Waite's
range reduction: the split is exact in fp32 for |x| < 2^22, and the power of two
goes into the exponent field). 2^f is approximated by the degree-4 polynomial
that minimises the largest relative error max |p(f) / 2^f - 1| on [-1/2, 1/2],
found with the Remez exchange algorithm in fp64 (Remez, 1934; the form for a
relative error weights each equation by 2^f). Prints the coefficients c0..c4
(p(f) = c0 + c1 f + ... + c4 f^4) rounded to fp32 and the error bound.

    python -m triangle_attention_b200.csrc.gen_exp2_poly
"""

from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    n = degree + 2
    # start from the Chebyshev extrema of the interval
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i: unknowns c0..c_d, E
        A = np.zeros((n, n))
        for k in range(degree + 1):
            A[:, k] = x ** k
        A[:, -1] = -((-1.0) ** np.arange(n)) * np.exp2(x)
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:-1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        idx = np.where(np.diff(np.sign(err)) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + int(np.argmax(np.abs(err[b0:b1]))) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) != n:
            break
        x = grid[ext]
    return c, float(np.max(np.abs(err)))


def coefficients_f32():
    c, _ = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 200001)
    err = np.polyval(c32.astype(np.float64)[::-1], grid) / np.exp2(grid) - 1.0
    return c32, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c32, bound = coefficients_f32()
    for k, v in enumerate(c32):
        print(f"c{k} = {float(v).hex()}  # {float(v):.9g}")
    print(f"max relative error on [-1/2, 1/2] with fp32 coefficients: {bound:.3e}")
