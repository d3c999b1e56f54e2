"""Fits the polynomial used by the FMA-pipe exp2 of the attention kernels.

Method: 2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2] (Cody-Waite
range reduction with one exact step, since n is an integer).  2^f is
approximated by a degree-d polynomial minimising the maximum RELATIVE error
on [-1/2, 1/2], found with the Remez exchange algorithm (equioscillation of
the weighted error at d+2 points).  The result is rounded to fp32 and the
relative error of the fp32 coefficients is reported.

    python fit_exp2_poly.py [degree]
"""
import sys

import numpy as np


def remez_relative(fn, deg, a, b, iters=30):
    """Minimax polynomial p of degree `deg` for fn on [a, b] w.r.t. the
    relative error (p - fn) / fn.  Returns (coefficients low->high, error)."""
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    grid = np.linspace(a, b, 200001)
    E = 0.0
    for _ in range(iters):
        # solve p(x_i) - fn(x_i) = (-1)^i E fn(x_i) for the coefficients and E
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * fn(x[i])
        sol = np.linalg.solve(A, fn(x))
        c, E = sol[:deg + 1], sol[deg + 1]
        err = (np.polyval(c[::-1], grid) - fn(grid)) / fn(grid)
        # new reference: the extrema of the error between its sign changes
        sgn = np.sign(err)
        idx = np.concatenate(([0], np.nonzero(np.diff(sgn))[0] + 1, [len(grid)]))
        ext = [s + np.argmax(np.abs(err[s:e])) for s, e in zip(idx[:-1], idx[1:]) if e > s]
        if len(ext) < n:
            break
        ext = np.array(ext)
        # keep n alternating extrema with the largest magnitudes
        while len(ext) > n:
            drop = 0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else len(ext) - 1
            ext = np.delete(ext, drop)
        x = grid[ext]
    err = (np.polyval(c[::-1], grid) - fn(grid)) / fn(grid)
    return c, float(np.abs(err).max())


def main():
    deg = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_relative(lambda t: np.exp2(t), deg, -0.5, 0.5)
    c32 = c.astype(np.float32)
    grid = np.linspace(-0.5, 0.5, 200001)
    f32 = (np.polyval(c32.astype(np.float64)[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
    print(f"degree {deg}: minimax relative error {e:.3e}, with fp32 coefficients "
          f"{np.abs(f32).max():.3e}")
    for i, v in enumerate(c32):
        print(f"  c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")


if __name__ == "__main__":
    main()
