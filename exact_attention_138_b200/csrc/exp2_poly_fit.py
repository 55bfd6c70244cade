"""Derivation of the degree-3 polynomial for 2^f, f in [-1/2, 1/2], used by the forward kernel to
compute part of the exponentials on the FMA pipe (fwd_bf16.cu, exp2_fma_x2).

Method: Remez exchange algorithm (E. Remez, 1934) for the minimax RELATIVE error, in fp64, then
the coefficients are rounded to fp32. The full exp2 is 2^x = 2^n · 2^f with n = round(x), the
Cody & Waite style reduction (W. J. Cody and W. Waite, "Software Manual for the Elementary
Functions", 1980). Run: python exp2_poly_fit.py  (prints the coefficients and the max relative
error of fp32 Horner evaluation, about 7.5e-5, far below bf16's 2^-9).
"""
import numpy as np


def remez_exp2(deg=3, a=-0.5, b=0.5, iters=50):
    f = np.exp2
    k = np.arange(deg + 2)
    xs = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * k / (deg + 1))[::-1]
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        A = np.zeros((deg + 2, deg + 2))
        for i, x in enumerate(xs):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f(x)
        sol = np.linalg.solve(A, f(xs))
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        idx = [0] + [i for i in range(1, len(grid) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        sel = []
        for x, e in zip(grid[idx], err[idx]):
            if sel and np.sign(e) == np.sign(sel[-1][1]):
                if abs(e) > abs(sel[-1][1]):
                    sel[-1] = (x, e)
            else:
                sel.append((x, e))
        while len(sel) > deg + 2:
            sel.pop(0 if abs(sel[0][1]) < abs(sel[-1][1]) else -1)
        xs = np.array([s[0] for s in sel])
    return c


if __name__ == "__main__":
    c = remez_exp2().astype(np.float32)
    g = np.linspace(-0.5, 0.5, 2000001).astype(np.float32)
    h = np.float32(c[3])
    for ci in c[2::-1]:
        h = np.float32(h * g + ci)
    rel = np.abs(h.astype(np.float64) - np.exp2(g.astype(np.float64))) / np.exp2(g.astype(np.float64))
    print("c0..c3 =", [float(x) for x in c], " max rel err =", rel.max())
