"""Fit the polynomial behind the FMA-pipe exp2 of the forward kernel.

2^x = 2^j * 2^f with j = round(x) and f = x - j in [-1/2, 1/2].  2^f is approximated by a
degree-n polynomial whose coefficients minimise the maximum RELATIVE error on [-1/2, 1/2]
(Remez exchange algorithm: solve p(x_i) = 2^x_i (1 + (-1)^i E) on n+2 alternation points,
move the points to the extrema of the error, repeat until the extrema equioscillate).
Run:  python fit_exp2.py [degree]   -> prints the coefficients c0..cn (float32) and the error.
"""
from __future__ import annotations

import sys

import numpy as np


def remez_exp2(n: int, iters: int = 30):
    lo, hi = -0.5, 0.5
    k = np.arange(n + 2)
    x = 0.5 * (lo + hi) + 0.5 * (hi - lo) * np.cos(np.pi * (n + 1 - k) / (n + 1))  # Chebyshev extrema
    grid = np.linspace(lo, hi, 200001)
    c = None
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        sign = np.sign(err)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        runs = np.split(np.arange(len(grid)), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n + 2:
            break
        while len(ext) > n + 2:  # drop the smallest end extremum
            ext = ext[1:] if abs(err[ext[0]]) < abs(err[ext[-1]]) else ext[:-1]
        x = grid[ext]
    err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
    return c, float(np.abs(err).max())


def exp2_poly_f32(x: np.ndarray, c) -> np.ndarray:
    """The kernel's arithmetic in float32: round-to-integer by the 1.5*2^23 shift, Horner in
    FMA order, exponent added in the integer domain."""
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    shift = np.float32(12582912.0)
    t = (x + shift).astype(np.float32)
    j = (t.view(np.int32) - np.int32(0x4B400000)).astype(np.int32)
    f = (x - (t - shift).astype(np.float32)).astype(np.float32)
    cf = [np.float32(v) for v in c]
    p = np.full_like(f, cf[-1])
    for v in cf[-2::-1]:
        p = (p * f + v).astype(np.float32)   # FMA rounding differs by < 1 ulp
    t_bits = t.view(np.int32).astype(np.int64)
    out = (p.view(np.int32).astype(np.int64) + (t_bits << 23)) & 0xFFFFFFFF   # the kernel's wrap-around form
    assert np.array_equal(out, (p.view(np.int32).astype(np.int64) + (j.astype(np.int64) << 23)) & 0xFFFFFFFF)
    return out.astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    n = int(sys.argv[1]) if len(sys.argv) > 1 else 3
    c, e = remez_exp2(n)
    print(f"degree {n}: max relative error {e:.3e} (2^{np.log2(e):.2f})")
    print("coefficients c0..cn (float32):", ", ".join(f"{float(np.float32(v)):.9g}f" for v in c))
    xs = np.linspace(-124, 8, 400001).astype(np.float32)
    rel = np.abs(exp2_poly_f32(xs, c).astype(np.float64) / np.exp2(xs.astype(np.float64)) - 1).max()
    print(f"float32 evaluation over [-124, 8]: max relative error {rel:.3e}")
    tail = exp2_poly_f32(np.array([-125.0, -126.0, -200.0, -np.inf], np.float32), c)
    assert np.all(np.isfinite(tail)) and np.all(tail >= 0) and np.all(tail < 1e-37), tail
    print("clamped tail (-125, -126, -200, -inf):", tail)
