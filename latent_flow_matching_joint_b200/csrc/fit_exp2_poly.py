"""Fit the polynomial used by the attention kernel's FMA-pipe exp2.

2^x is split as 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2];
2^f is approximated by a cubic c0 + c1 f + c2 f^2 + c3 f^3 chosen to minimise
the maximum relative error on [-1/2, 1/2] (a small Remez exchange started from
a Chebyshev least-squares fit). Prints the coefficients (float32) and the
achieved maximum relative error, evaluated in float32 Horner form exactly as
the kernel does.
"""
import numpy as np


def remez_rel(deg=3, a=-0.5, b=0.5, iters=30):
    # initial reference: Chebyshev extrema
    k = np.arange(deg + 2)
    xs = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * k / (deg + 1))[::-1]
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  (equioscillating relative error)
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        c = sol[:deg + 1]
        grid = np.linspace(a, b, 200001)
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: local extrema of the error, one per sign change interval
        idx = np.where(np.diff(np.sign(np.diff(err))) != 0)[0] + 1
        cand = np.concatenate([[0], idx, [len(grid) - 1]])
        if len(cand) >= deg + 2:
            # keep the deg+2 largest alternating extrema
            vals = err[cand]
            order = np.argsort(-np.abs(vals))[:deg + 2]
            xs = np.sort(grid[cand[order]])
    return c


def horner_f32(c, f):
    c = c.astype(np.float32)
    f = f.astype(np.float32)
    p = c[3]
    p = np.float32(p) * f + c[2]
    p = p * f + c[1]
    p = p * f + c[0]
    return p.astype(np.float32)


if __name__ == "__main__":
    c = remez_rel().astype(np.float32)
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    rel = np.abs(horner_f32(c, f).astype(np.float64) - 2.0 ** f.astype(np.float64)) / 2.0 ** f.astype(np.float64)
    for i, v in enumerate(c):
        print(f"c{i} = {float(v)!r}f")
    print(f"max relative error (float32 Horner on [-1/2, 1/2]) = {rel.max():.3e}")
