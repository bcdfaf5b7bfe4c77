"""Coefficients of the polynomial 2^f ~ P(f), f in [-1/2, 1/2], used by
ex2_poly() in ptx.cuh to compute part of the exponentials on the FMA pipe.

Method: the Remez exchange algorithm (E. Ya. Remez, 1934) for the best
approximation in the RELATIVE error |P(f) / 2^f - 1| of a degree-5 polynomial
on [-1/2, 1/2]: solve for the polynomial that equioscillates on n + 2 reference
points, move the references to the extrema of the new error curve, repeat.
The coefficients are then rounded to float32; the script reports the maximum
relative error of the rounded polynomial on a dense grid (float64 evaluation).

    python lm_head_projection_supervised_b200/csrc/exp2_poly_fit.py
"""
import numpy as np

DEG = 5
A, B = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    k = np.arange(n)
    x = 0.5 * (A + B) + 0.5 * (B - A) * np.cos(np.pi * (n - 1 - k) / (n - 1))  # Chebyshev extrema
    grid = np.linspace(A, B, 200001)
    for _ in range(iters):
        f = np.exp2(x)
        M = np.zeros((n, n))
        M[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        M[:, deg + 1] = ((-1.0) ** k) * f  # relative-error weight
        sol = np.linalg.solve(M, f)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / np.exp2(grid) - 1.0
        # one extremum per sign run of the error curve
        s = np.sign(err)
        runs = np.flatnonzero(np.diff(s) != 0) + 1
        bounds = np.concatenate([[0], runs, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:])]
        if len(ext) < n:
            break
        # keep the n largest consecutive alternating extrema
        ext = np.array(ext)
        while len(ext) > n:
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        x = grid[ext]
    return c


def main():
    c = remez()
    c32 = c.astype(np.float32)
    g = np.linspace(A, B, 2000001)
    rel = np.abs(np.polyval(c32.astype(np.float64)[::-1], g) / np.exp2(g) - 1.0)
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v).hex()}  ({float(v):.9g})")
    print(f"max relative error of the float32-rounded polynomial: {rel.max():.3e}")


if __name__ == "__main__":
    main()
