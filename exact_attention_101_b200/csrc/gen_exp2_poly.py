"""Fit the cubic used for the software base-2 exponential in fa_fwd_kernel.cuh.

The kernel evaluates 2^x as 2^j * p(f) with j = round(x), f = x - j in [-1/2, 1/2]
(Cody-Waite style range reduction) and p a degree-3 polynomial.  This script computes
the minimax p for RELATIVE error on [-1/2, 1/2] with the Remez exchange algorithm
(equioscillation of the weighted error at deg+2 points), prints the coefficients as
fp32 literals and the achieved maximum relative error.

    python gen_exp2_poly.py
"""
import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg=DEG, iters=30):
    n = deg + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    x = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k / (n - 1))[::-1]
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        f = 2.0 ** x
        # p(x_i) - f(x_i) = (-1)^i E f(x_i)   (relative error equioscillates)
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * f[i]
        sol = np.linalg.solve(A, f)
        c = sol[:deg + 1]
        err = (np.polyval(c[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extrema of the error between sign changes
        idx = [0]
        for i in range(1, len(grid) - 1):
            if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0:
                idx.append(i)
        idx.append(len(grid) - 1)
        cand = np.array(idx)
        # keep the n largest alternating extrema
        sel = []
        for i in cand:
            if sel and np.sign(err[i]) == np.sign(err[sel[-1]]):
                if abs(err[i]) > abs(err[sel[-1]]):
                    sel[-1] = i
            else:
                sel.append(i)
        while len(sel) > n:
            if abs(err[sel[0]]) < abs(err[sel[-1]]):
                sel.pop(0)
            else:
                sel.pop()
        x = grid[np.array(sel)]
    return c, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    g = np.linspace(LO, HI, 400001)
    e32 = np.max(np.abs((np.polyval(c32.astype(np.float64)[::-1], g) - 2.0 ** g) / 2.0 ** g))
    for i, v in enumerate(c32):
        print("c%d = %.9ef" % (i, v))
    print("max relative error: %.3e (float64 coefficients), %.3e (fp32 coefficients)" % (e, e32))
