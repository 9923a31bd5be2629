"""Coefficients of the polynomial 2^f used for part of the softmax exponentials.

The softmax of the tensor-core attention evaluates exp2 on the MUFU unit (16 results per
clock per SM), which caps head_dim 64 at about half the tensor-core rate.  Part of the
exponentials therefore run on the FMA pipe instead: x = n + f with n = round(x) and
f in [-1/2, 1/2]; 2^x = 2^n * p(f), where p is the degree-3 polynomial that minimises the
maximum relative error |p(f) / 2^f - 1| on [-1/2, 1/2] (Remez exchange, Chebyshev
alternation: the error equioscillates at degree + 2 points), and 2^n is added to the
exponent bits of p(f).

Run: python long_video_diffusion_b200/csrc/fit_exp2_poly.py  -> prints the coefficients
(c0 + c1 f + c2 f^2 + c3 f^3, as float32 hex and decimal) and the error bound, which
tests/test_exp2_poly.py checks against the constants in dp_attn_tc.cu.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(nodes: np.ndarray) -> tuple[np.ndarray, float]:
    # p(x_i) - 2^x_i = (-1)^i E 2^x_i   (relative error alternates with amplitude E)
    n = nodes.size
    A = np.zeros((n, DEGREE + 2))
    for k in range(DEGREE + 1):
        A[:, k] = nodes ** k
    A[:, DEGREE + 1] = -((-1.0) ** np.arange(n)) * np.exp2(nodes)
    sol = np.linalg.solve(A, np.exp2(nodes))
    return sol[:DEGREE + 1], float(sol[DEGREE + 1])


def _rel_err(c: np.ndarray, x: np.ndarray) -> np.ndarray:
    p = np.polynomial.polynomial.polyval(x, c)
    return p / np.exp2(x) - 1.0


def remez(iters: int = 30):
    k = np.arange(DEGREE + 2)
    nodes = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (DEGREE + 1 - k) / (DEGREE + 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(nodes)
        e = _rel_err(c, grid)
        # new nodes: the extremum of e on each interval between sign changes (plus ends)
        s = np.sign(e)
        cuts = np.flatnonzero(np.diff(s) != 0) + 1
        pieces = np.split(np.arange(grid.size), cuts)
        ext = np.array([p[np.argmax(np.abs(e[p]))] for p in pieces if p.size])
        if ext.size != DEGREE + 2:
            break
        nodes = grid[ext]
    return c, float(np.max(np.abs(_rel_err(c, grid))))


def float32_coeffs():
    c, err = remez()
    c32 = c.astype(np.float32)
    grid = np.linspace(LO, HI, 200001)
    err32 = float(np.max(np.abs(_rel_err(c32.astype(np.float64), grid))))
    return c32, err, err32


if __name__ == "__main__":
    c32, err, err32 = float32_coeffs()
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v)!r:24s} 0x{np.float32(v).view(np.uint32):08x}")
    print(f"max relative error: {err:.3e} (float64 coefficients), {err32:.3e} (float32 coefficients)")
