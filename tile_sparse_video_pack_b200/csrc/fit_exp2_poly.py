"""Fits the degree-4 polynomial for 2^f, f in [-1/2, 1/2], used by the attention kernel.

The kernel computes part of its exponentials on the FMA pipe (ex2_fma_pipe in
attn.cu): x = n + f with n = round(x), 2^x = 2^n * P(f). P minimises the
maximum RELATIVE error |P(f) / 2^f - 1| over [-1/2, 1/2]; it is found by the
Remez exchange algorithm (E. Ya. Remez, 1934): solve for the polynomial whose
relative error equioscillates on deg + 2 reference points, move the reference
to the extrema of the new error curve, repeat.

    python tile_sparse_video_pack_b200/csrc/fit_exp2_poly.py

prints the fp32 coefficients (lowest degree first) and the maximum relative
error of the polynomial evaluated in fp32 by Horner's rule.
"""
from __future__ import annotations

import numpy as np


def remez_exp2(deg: int = 4, a: float = -0.5, b: float = 0.5, iters: int = 40):
    n = deg + 2
    x = np.sort((a + b) / 2 + (b - a) / 2 * np.cos(np.pi * np.arange(n) / (n - 1)))
    grid = np.linspace(a, b, 200001)
    f = np.exp2
    c = None
    for _ in range(iters):
        A = np.zeros((n, n))
        A[:, :deg + 1] = x[:, None] ** np.arange(deg + 1)[None, :]
        A[:, deg + 1] = (-1.0) ** np.arange(n) * f(x)
        sol = np.linalg.solve(A, f(x))
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / f(grid) - 1.0
        # one extremum per run of constant sign
        sign = np.sign(err)
        cuts = np.nonzero(np.diff(sign) != 0)[0] + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = np.array([s[np.argmax(np.abs(err[s]))] for s in segs])
        if ext.size != n:
            break
        x = grid[ext]
    return c


def horner_f32(coeffs32: np.ndarray, f: np.ndarray) -> np.ndarray:
    p = np.full_like(f, coeffs32[-1])
    for ci in coeffs32[-2::-1]:
        p = (p * f + ci).astype(np.float32)
    return p


def fit(deg: int = 4):
    c32 = remez_exp2(deg).astype(np.float32)
    f = np.linspace(-0.5, 0.5, 1000001).astype(np.float32)
    err = np.max(np.abs(horner_f32(c32, f).astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0))
    return c32, float(err)


if __name__ == "__main__":
    c, e = fit()
    print("coefficients (f^0 .. f^4):", [repr(float(v)) for v in c])
    print("max relative error in fp32:", e)
