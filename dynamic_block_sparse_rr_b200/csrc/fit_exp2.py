"""Fit the coefficients of the FMA-pipe exp2 used by the attention softmax.

2^x is split as 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2]; 2^f
is approximated by a polynomial whose coefficients minimise the maximum
relative error on [-1/2, 1/2] (Remez exchange with weight 2^-f).  Prints the
coefficients (lowest degree first) and the achieved error bound.

    python dynamic_block_sparse_rr_b200/csrc/fit_exp2.py [degree]
"""
import sys

import numpy as np


def remez_exp2(deg: int, iters: int = 40):
    lo, hi = -0.5, 0.5
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = -((-1.0) ** k) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** x)
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extremum of each sign-alternating segment
        sign = np.sign(err)
        bounds = np.nonzero(np.diff(sign) != 0)[0]
        segs = np.split(np.arange(grid.size), bounds + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) < n:
            break
        while len(ext) > n:  # drop the smaller end extremum
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        x = grid[ext]
    err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
    return c, float(np.max(np.abs(err))), abs(E)


if __name__ == "__main__":
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, emax, E = remez_exp2(deg)
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 100001)
    p32 = np.zeros_like(grid, dtype=np.float32)
    for ci in c32[::-1]:
        p32 = p32 * grid.astype(np.float32) + ci
    e32 = np.max(np.abs(p32.astype(np.float64) / 2.0 ** grid - 1.0))
    print(f"degree {deg}: max rel error {emax:.3e} (equioscillation {E:.3e}), as fp32 Horner {e32:.3e}")
    print("coefficients c0..c%d:" % deg)
    for ci in c32:
        print(f"  {float(ci):.9e}f  ({float(ci).hex()})")
