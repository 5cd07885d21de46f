"""Coefficients of the polynomial 2^f used by the attention kernels for part of
their exponentials (kept off the special-function unit).

Method: Cody-Waite range reduction x = n + f with n = round(x) and f in
[-1/2, 1/2], so 2^x = 2^n * 2^f; 2^f is approximated by the degree-3
polynomial that minimises the maximum RELATIVE error on [-1/2, 1/2], found by
the Remez exchange algorithm (equioscillation at deg + 2 points); 2^n is
applied by adding n to the float's exponent field.

Running this file prints the coefficients (as C float literals) and the
maximum relative error over a fine grid; the kernel's constants were pasted
from its output.
"""
import numpy as np


def remez_exp2(deg=3, a=-0.5, b=0.5, iters=40):
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 400001)
    for _ in range(iters):
        # solve p(x_i) / 2^x_i - 1 = (-1)^i E for the coefficients and E
        A = np.zeros((n, n))
        for k in range(deg + 1):
            A[:, k] = x ** k / np.exp2(x)
        A[:, -1] = (-1.0) ** np.arange(n)
        sol = np.linalg.solve(A, np.ones(n))
        c = sol[:-1]
        err = np.polynomial.polynomial.polyval(grid, c) / np.exp2(grid) - 1.0
        # new reference: alternating extrema of the error curve
        ext = [0] + [i for i in range(1, len(grid) - 1)
                     if (err[i] - err[i - 1]) * (err[i + 1] - err[i]) <= 0] + [len(grid) - 1]
        pts = []
        for i in ext:
            if pts and np.sign(err[i]) == np.sign(err[pts[-1]]):
                if abs(err[i]) > abs(err[pts[-1]]):
                    pts[-1] = i
            else:
                pts.append(i)
        while len(pts) > n:
            pts.pop(0 if abs(err[pts[0]]) < abs(err[pts[-1]]) else -1)
        if len(pts) == n:
            x = grid[pts]
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_exp2()
    c32 = np.asarray(c, dtype=np.float32)
    grid = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    p = ((c32[3] * grid + c32[2]) * grid + c32[1]) * grid + c32[0]
    e32 = float(np.max(np.abs(p.astype(np.float64) / np.exp2(grid.astype(np.float64)) - 1.0)))
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r}f  ({v.view(np.uint32):#010x})")
    print(f"max relative error: {e:.3e} (float64 coefficients), {e32:.3e} (float32 Horner)")
