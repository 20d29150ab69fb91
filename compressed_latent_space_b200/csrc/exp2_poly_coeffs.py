"""Coefficients of the cubic that the latent attention evaluates 2^f with on the FMA pipes.

The minimax polynomial of degree 3 for 2^f on [-1/2, 1/2] under relative error, found by the
Remez exchange algorithm (solve for the coefficients and the levelled error on n + 2 reference
points, move the references to the extrema of the error, repeat).  ``common.cuh``'s
``ex2_poly2`` holds these numbers rounded to float; ``tests/test_exp2_poly.py`` re-derives
them and checks the source and the float32 error bound.  Run as a script to print them.
"""
import numpy as np


def remez_exp2(deg: int = 3, lo: float = -0.5, hi: float = 0.5, iters: int = 30):
    """Returns (coefficients c_0..c_deg, levelled relative error)."""
    n = deg + 2
    xs = np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (hi - lo) / 2 + (hi + lo) / 2
    grid = np.linspace(lo, hi, 200001)
    for _ in range(iters):
        a = np.zeros((n, n))
        for i, x in enumerate(xs):
            a[i, :deg + 1] = x ** np.arange(deg + 1)
            a[i, deg + 1] = (-1) ** i * np.exp2(x)
        sol = np.linalg.solve(a, np.exp2(xs))
        c, e = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        segs = np.split(np.arange(len(grid)), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs]
        if len(ext) != n:
            break
        xs = grid[ext]
    return c, abs(e)


if __name__ == "__main__":
    c, e = remez_exp2()
    print("c0..c3 =", ", ".join(f"{v:.9g}f" for v in np.float32(c)), f" (levelled relative error {e:.3g})")
