"""Derives the polynomial used by the kernels' FMA-pipe exp2.

The kernels evaluate 2^x for x <= 0 as 2^j * p(f) with j = rint(x) and
f = x - j in [-1/2, 1/2] (Cody-Waite range reduction), then add j to the
exponent field of p(f).  p is the degree-3 polynomial that minimises the
maximum RELATIVE error |p(f) / 2^f - 1| on [-1/2, 1/2], found here with the
Remez exchange algorithm in float64 and then rounded to float32.

Run:  python gen_exp2_poly.py      (prints the coefficients and error bounds)
"""
from __future__ import annotations

import numpy as np

DEG = 3
LO, HI = -0.5, 0.5


def remez(deg: int = DEG, iters: int = 30):
    n = deg + 2
    # start from Chebyshev extrema mapped to [LO, HI]
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n - 1 - k) / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(ref_i) - 2^ref_i = (-1)^i E 2^ref_i  ->  linear in (c_0..c_deg, E)
        A = np.zeros((n, n))
        for i, f in enumerate(ref):
            A[i, :deg + 1] = f ** np.arange(deg + 1)
            A[i, deg + 1] = -((-1) ** i) * 2.0 ** f
        sol = np.linalg.solve(A, 2.0 ** ref)
        c = sol[:deg + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the n alternating extrema of the error
        sgn = np.sign(err)
        cuts = np.flatnonzero(np.diff(sgn) != 0) + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = [s[np.argmax(np.abs(err[s]))] for s in segs if s.size]
        if len(ext) < n:
            break
        # keep n consecutive extrema with the largest error
        ext = np.array(ext)
        best = max(range(len(ext) - n + 1), key=lambda i: np.min(np.abs(err[ext[i:i + n]])))
        ref = grid[ext[best:best + n]]
    return c, float(np.max(np.abs(err)))


def f32_horner(c32, f):
    """fp32 Horner with fused multiply-adds (one rounding each), as on the GPU."""
    f = f.astype(np.float32)
    p = np.float32(c32[-1])
    for ci in c32[-2::-1]:
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(ci)).astype(np.float32)
    return p


def main():
    c, e = remez()
    c32 = np.array(c, dtype=np.float32)
    f = np.linspace(LO, HI, 400001).astype(np.float32)
    rel = f32_horner(c32, f).astype(np.float64) / 2.0 ** f.astype(np.float64) - 1.0
    print(f"degree {DEG} minimax relative error (float64 coefficients): {e:.3e}")
    print(f"max relative error with float32 coefficients and fp32 Horner: {np.max(np.abs(rel)):.3e}")
    for i, ci in enumerate(c32):
        print(f"c{i} = {float(ci).hex()}  ({float(ci):.9g})")


if __name__ == "__main__":
    main()
