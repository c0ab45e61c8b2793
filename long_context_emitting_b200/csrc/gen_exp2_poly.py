"""Generator of the kExp2Deg5 coefficients in exp2_poly.cuh.

The polynomial p(f) ~ 2^f on [-1/2, 1/2] minimises the maximum RELATIVE error
(p(f) - 2^f) / 2^f.  It is found with the Remez exchange algorithm: start
from the Chebyshev extrema as the reference set; on each pass solve the linear
system p(x_i) - 2^x_i = (-1)^i E 2^x_i for the coefficients and the levelled
error E; then take as the new reference the point of largest |error| in each
interval between sign changes of the error on a fine grid.  The float64
result is rounded to float32 for the header.

  python -m long_context_emitting_b200.csrc.gen_exp2_poly   (prints the header line)
"""
from __future__ import annotations

import numpy as np

LO, HI = -0.5, 0.5
GRID = 200001


def remez_exp2(degree: int, iters: int = 40):
    """(float64 coefficients lowest order first, max relative error on the grid)."""
    n = degree + 2
    x = (np.cos(np.pi * np.arange(n) / (n - 1))[::-1] * (HI - LO) + (HI + LO)) / 2
    grid = np.linspace(LO, HI, GRID)
    err = None
    c = None
    for _ in range(iters):
        a = np.zeros((n, n))
        for i in range(n):
            a[i, :degree + 1] = x[i] ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * np.exp2(x[i])
        sol = np.linalg.solve(a, np.exp2(x))
        c = sol[:degree + 1]
        err = (np.polyval(c[::-1], grid) - np.exp2(grid)) / np.exp2(grid)
        segs = np.split(np.arange(GRID), np.where(np.diff(np.sign(err)) != 0)[0] + 1)
        x = np.array([grid[s[np.argmax(np.abs(err[s]))]] for s in segs])
        if len(x) != n:  # keep n alternating extrema
            x = x[:n] if len(x) > n else np.concatenate([x, [HI] * (n - len(x))])
    return c, float(np.abs(err).max())


def float32_coefficients(degree: int = 5):
    c, _ = remez_exp2(degree)
    return [float(np.float32(v)) for v in c]


if __name__ == "__main__":
    cs = float32_coefficients(5)
    print("constexpr float kExp2Deg5[6] = {" + ", ".join(f"{v!r}f" for v in cs) + "};")
