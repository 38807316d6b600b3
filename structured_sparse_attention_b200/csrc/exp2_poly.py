"""Coefficients of the FMA-pipe exp2 of the kernels (common.cuh, exp2_fma2).

Method (Cody and Waite, "Software Manual for the Elementary Functions", 1980: argument
reduction; Remez exchange for the minimax fit):
  2^x = 2^n * 2^f,  n = round-to-nearest(x),  f = x - n in [-1/2, 1/2]
  2^f ~= c0 + c1 f + c2 f^2 + c3 f^3 + c4 f^4, minimax in RELATIVE error on [-1/2, 1/2]
  2^n is applied by adding n to the exponent field of the polynomial's value.

Run this file to print the coefficients (rounded to fp32) and the error bounds; the
kernels' constants (common.cuh, kExp2C*) are its output, and a CPU test checks that
they agree and that the fp32 evaluation meets the bound.
"""

from __future__ import annotations

import numpy as np

DEGREE = 4
LO, HI = -0.5, 0.5


def remez(deg: int = DEGREE, a: float = LO, b: float = HI, iters: int = 40, grid_n: int = 200001):
    """Minimax polynomial (ascending coefficients) for 2^f on [a, b], relative error."""
    n = deg + 2
    ref = (a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n) / (n - 1))[::-1]
    grid = np.linspace(a, b, grid_n)
    fg = np.exp2(grid)
    coef = None
    for _ in range(iters):
        A = np.zeros((n, n))
        fx = np.exp2(ref)
        for i, x in enumerate(ref):
            A[i, :deg + 1] = x ** np.arange(deg + 1)
            A[i, deg + 1] = (-1) ** i * fx[i]
        coef = np.linalg.solve(A, fx)[:deg + 1]
        err = (np.polyval(coef[::-1], grid) - fg) / fg
        # local extrema of the error, merged into runs of alternating sign
        d = np.diff(err)
        ext = [0] + [i for i in range(1, grid_n - 1) if d[i - 1] * d[i] <= 0] + [grid_n - 1]
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
            ref = grid[pts]
    return coef


def coefficients_f32() -> np.ndarray:
    return remez().astype(np.float32)


def emulate(x: np.ndarray, c: np.ndarray) -> np.ndarray:
    """The kernel's fp32 evaluation, step for step (x clamped to >= -126)."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23: x + magic rounds x to an integer
    t = (x + magic).astype(np.float32)
    nn = (t - magic).astype(np.float32)
    f = (x - nn).astype(np.float32)
    p = np.full_like(f, c[-1])
    for k in range(len(c) - 2, -1, -1):
        p = (p * f + c[k]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c = coefficients_f32()
    g = np.linspace(LO, HI, 1000001).astype(np.float32)
    p = emulate(g, c).astype(np.float64)
    rel = np.abs(p / np.exp2(g.astype(np.float64)) - 1).max()
    print(f"degree {DEGREE}: max relative error of the fp32 evaluation on [-1/2, 1/2]: {rel:.3e}")
    for k, v in enumerate(c):
        print(f"constexpr float kExp2C{k} = {float(v)!r}f;")
