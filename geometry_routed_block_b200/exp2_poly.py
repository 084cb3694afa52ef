"""Coefficients of the degree-3 polynomial the attention kernel uses for part
of its base-2 exponentials (the rest go to the hardware ex2 unit).

Method: Cody-Waite range reduction -- 2^x = 2^n * 2^f with n = round(x) and
f = x - n in [-1/2, 1/2] -- and a minimax polynomial p(f) ~ 2^f for the
relative error, found with the Remez exchange algorithm. The kernel evaluates
p in float32 with fused multiply-adds (Horner) and adds n to the exponent field
of p(f). The polynomial's relative error bound is about 7.5e-5, far below the
bf16 rounding (2^-9) the probabilities then go through.

    python -m geometry_routed_block_b200.exp2_poly   # prints the coefficients
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(deg: int = DEGREE, a: float = LO, b: float = HI, iters: int = 30):
    """Minimax polynomial for 2^x on [a, b] in the relative-error sense.
    Returns (coefficients c0..c_deg in float64, max relative error)."""
    f = np.exp2
    n = deg + 2
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        for i in range(n):
            A[i, : deg + 1] = x[i] ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * f(x[i])
        sol = np.linalg.solve(A, f(x))
        c = sol[: deg + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        sign = np.sign(err)
        ext, start = [], 0
        for k in range(1, len(grid) + 1):
            if k == len(grid) or sign[k] != sign[start]:
                seg = np.arange(start, k)
                ext.append(seg[np.argmax(np.abs(err[seg]))])
                start = k
        ext = np.array(ext)
        while len(ext) > n:
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        x = grid[ext]
    err = np.polyval(c[::-1], grid) / f(grid) - 1.0
    return c, float(np.abs(err).max())


def coefficients_f32():
    c, _ = remez_relative()
    return [float(np.float32(v)) for v in c]


if __name__ == "__main__":
    c, e = remez_relative()
    print("coefficients (c0..c3):", [float(np.float32(v)) for v in c], "max rel err", e)
