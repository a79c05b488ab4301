"""Fits the polynomial behind the FMA-pipe exp2 of the attention kernel.

The kernel (csrc/attn_device.cuh, ``exp2_poly_x2``) computes 2^x as 2^j * p(f)
with j = rint(x) and f = x - j in [-1/2, 1/2].  p is the degree-3 polynomial
with the smallest maximum relative error to 2^f on that interval, found
here by the Remez exchange algorithm; the kernel's constants kPc0..kPc3 are
its coefficients rounded to float32.

Usage: ``python -m kv_cached_segment_b200.fit_exp2_poly`` prints them.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(degree: int = 3, a: float = -0.5, b: float = 0.5, iters: int = 30):
    """Coefficients (lowest power first) and the minimax relative error."""
    n = degree + 2
    # start from the Chebyshev extrema of the interval
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * np.arange(n)[::-1] / (n - 1))
    grid = np.linspace(a, b, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i: equal relative error of alternating sign
        m = np.zeros((n, n))
        for i in range(n):
            m[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            m[i, degree + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(m, np.exp2(x))
        coef = sol[:degree + 1]
        err = (np.polyval(coef[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        # next reference: the extremum of each run of constant sign
        runs = np.split(np.arange(grid.size), np.nonzero(np.diff(np.sign(err)))[0] + 1)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) >= n:
            ext = ext if len(ext) == n else sorted(ext, key=lambda i: -abs(err[i]))[:n]
            x = np.sort(grid[ext])
    return coef, float(np.max(np.abs(err)))


if __name__ == "__main__":
    coef, err = remez_exp2()
    for k, c in enumerate(coef.astype(np.float32)):
        print(f"constexpr float kPc{k} = {float(c)!r}f;")
    print(f"// minimax relative error {err:.3e}")
