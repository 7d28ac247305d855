"""Fit the polynomial used by the attention kernel's FMA-pipe exp2 (run: python fit_exp2_poly.py).

Method: 2^x = 2^n * 2^f with n = round(x) and f = x - n in [-1/2, 1/2] (Cody-Waite style range
reduction for base 2, exact in floating point), and 2^f approximated by the degree-3
polynomial that minimises the maximum *relative* error on [-1/2, 1/2], found with the Remez
exchange algorithm.  Prints the float32 coefficients (c0..c3) and the achieved error, which
the kernel's constants and the emulation test reproduce.
"""
import numpy as np

DEG, A, B = 3, -0.5, 0.5


def remez(deg=DEG, a=A, b=B, iters=30):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    coef = None
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative equioscillation)
        M = np.zeros((n, n))
        for i in range(n):
            M[i, :deg + 1] = x[i] ** np.arange(deg + 1)
            M[i, deg + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(M, 2.0 ** x)
        coef = sol[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
        # new reference: the extremum of the error in each sign-constant segment
        sign_change = np.flatnonzero(np.diff(np.sign(err))) + 1
        segments = np.split(np.arange(grid.size), sign_change)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments]
        if len(ext) < n:
            break
        ext = sorted(ext, key=lambda k: -abs(err[k]))[:n]
        x = np.sort(grid[ext])
    err = (np.polyval(coef[::-1], grid) - 2.0 ** grid) / 2.0 ** grid
    return coef, np.max(np.abs(err))


if __name__ == "__main__":
    c, e = remez()
    c32 = c.astype(np.float32)
    g = np.linspace(A, B, 200001)
    e32 = np.max(np.abs((np.polyval(c32.astype(np.float64)[::-1], g) - 2.0 ** g) / 2.0 ** g))
    print("coefficients c0..c3 (float32):", ", ".join(f"{v:.9e}f" for v in c32))
    print(f"max relative error: {e:.3e} (exact coefficients), {e32:.3e} (float32 coefficients)")
