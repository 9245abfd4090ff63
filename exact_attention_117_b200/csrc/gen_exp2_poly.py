"""Derives the cubic used by exp2_poly3 (sm100.cuh) for 2^f on [-0.5, 0.5].

Remez exchange for the minimax RELATIVE error of a degree-3 polynomial:
solve p(x_i) + (-1)^i E 2^{x_i} = 2^{x_i} on n+2 reference points, move the
points to the extrema of the error, repeat.  Prints the float32 coefficients
c0..c3 and the maximum relative error.  Not run at build time; the printed
values are written into sm100.cuh.
"""
import numpy as np


def remez_exp2(deg=3, a=-0.5, b=0.5, iters=40, grid=200001):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n) / (n - 1))[::-1]
    g = np.linspace(a, b, grid)
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * np.exp2(x[i])
        sol = np.linalg.solve(A, np.exp2(x))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], g) - np.exp2(g)) / np.exp2(g)
        d = np.diff(err)
        cand = np.concatenate([[0], np.where(d[:-1] * d[1:] <= 0)[0] + 1, [grid - 1]])
        pts = []
        for k in cand:
            if pts and np.sign(err[k]) == np.sign(err[pts[-1]]):
                if abs(err[k]) > abs(err[pts[-1]]):
                    pts[-1] = k
            else:
                pts.append(k)
        while len(pts) > n:
            if abs(err[pts[0]]) < abs(err[pts[-1]]):
                pts.pop(0)
            else:
                pts.pop()
        if len(pts) < n:
            break
        x = g[pts]
    return c.astype(np.float32), float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_exp2()
    print("c0..c3 =", [float(v) for v in c], "max relative error = %.3e" % e)
