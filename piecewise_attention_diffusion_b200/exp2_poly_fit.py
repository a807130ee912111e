"""Fit of the polynomial that the forward kernel uses for part of its exponentials.

The softmax of the forward kernel evaluates 2^x for x <= 8. Most values go through the
special-function unit (ex2); a fixed share is computed on the FMA pipe instead so that
both pipes work in parallel. That path uses a Cody-Waite style split x = n + f with
n = rint(x) and f in [-1/2, 1/2] (W. J. Cody and W. Waite, "Software Manual for the
Elementary Functions", 1980), evaluates 2^f with a degree-3 polynomial and adds n to the
exponent field. The polynomial minimises the maximum RELATIVE error of p(f) against 2^f
on [-1/2, 1/2]; its coefficients come from the Remez exchange below (float64), rounded to
float32. Run this file to reproduce them:

    python -m piecewise_attention_diffusion_b200.exp2_poly_fit
"""
import numpy as np


def remez_exp2(degree: int = 3, iters: int = 30, grid: int = 200001):
    a, b = -0.5, 0.5
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(degree + 2)[::-1] / (degree + 1))
    g = np.linspace(a, b, grid)
    for _ in range(iters):
        A = np.zeros((degree + 2, degree + 2))
        for i in range(degree + 2):
            A[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], g) - 2.0 ** g) / 2.0 ** g
        ext, start, sign = [], 0, np.sign(err)
        for i in range(1, grid):
            if sign[i] != sign[start]:
                ext.append(start + int(np.argmax(np.abs(err[start:i]))))
                start = i
        ext.append(start + int(np.argmax(np.abs(err[start:]))))
        while len(ext) > degree + 2:
            ext.pop(0 if abs(err[ext[0]]) < abs(err[ext[-1]]) else -1)
        if len(ext) == degree + 2:
            x = g[ext]
    return c, float(np.abs(err).max())


if __name__ == "__main__":
    c, e = remez_exp2(3)
    print(f"max relative error {e:.3e}")
    for k, v in enumerate(c):
        print(f"c{k} = {np.float32(v)!r}  (0x{np.float32(v).view(np.uint32):08x})")
