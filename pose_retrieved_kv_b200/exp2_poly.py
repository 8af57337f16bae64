"""Coefficients of the polynomial exp2 used for part of the softmax exponentials.

The attention kernel's softmax needs 2^x for every score; the special-function unit gives 16
results per clock per SM, which is exactly the rate the tensor cores consume scores at, so a
share of the exponentials is computed on the FMA pipe instead, by Cody-Waite range reduction
(Cody and Waite, "Software Manual for the Elementary Functions", 1980): x = n + f with n the
nearest integer (taken with the 1.5 * 2^23 rounding constant) and f in [-1/2, 1/2], then
2^x = 2^f * 2^n with 2^n added to the exponent field of p(f), p a degree-3 polynomial that
minimises the maximum RELATIVE error of p(f) against 2^f on [-1/2, 1/2].  This script finds p
by the Remez exchange algorithm (equioscillation of the weighted error on five reference points)
and prints the float32 coefficients the kernel holds.  The weights are rounded to bf16 (8
significant bits) right after, so a relative error near 1e-4 is far below what that rounding
adds (2^-9).

Usage: ``python pose_retrieved_kv_b200/exp2_poly.py``.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
CLAMP = -125.0        # n >= -125 keeps the exponent field of p(f) * 2^n positive
LO, HI = -0.5, 0.5


def remez(degree: int = DEGREE, iters: int = 30):
    """Coefficients c[0..degree] (ascending powers) and the levelled relative error."""
    n = degree + 2
    # start from Chebyshev extrema
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * -np.cos(np.pi * k / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    for _ in range(iters):
        # p(x_i) - 2^x_i = (-1)^i E 2^x_i  (relative error levelled at E)
        a = np.zeros((n, n))
        for i, x in enumerate(ref):
            a[i, :degree + 1] = x ** np.arange(degree + 1)
            a[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(a, 2.0 ** ref)
        c, e = sol[:degree + 1], sol[degree + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: one extremum of the error per sign run
        sgn = np.sign(err)
        cuts = np.flatnonzero(np.diff(sgn) != 0) + 1
        runs = np.split(np.arange(len(grid)), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) != n:
            break
        ref = grid[ext]
    return c, abs(e)


def coefficients_f32():
    c, _ = remez()
    return [np.float32(v) for v in c]


def exp2_emulated(x: np.ndarray) -> np.ndarray:
    """The kernel's arithmetic in float32 (numpy does not fuse the multiply-adds; the kernel's
    fma rounds once per step, which only improves on this): clamp below at CLAMP, round with
    the 1.5 * 2^23 constant, Horner, add n to the exponent field.  Below -125 the result is
    2^-125 instead of (nearly) 0: negligible next to the row sum, which is >= 1."""
    c = coefficients_f32()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(CLAMP))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    r = (t - magic).astype(np.float32)
    f = (x - r).astype(np.float32)
    p = c[3]
    for ci in (c[2], c[1], c[0]):
        p = (p * f + ci).astype(np.float32)
    bits = p.view(np.uint32).astype(np.uint64) + (t.view(np.uint32).astype(np.uint64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


if __name__ == "__main__":
    c, e = remez()
    print(f"levelled relative error {e:.3e}")
    for i, v in enumerate(coefficients_f32()):
        print(f"c{i} = {float(v)!r}f  (0x{np.float32(v).view(np.uint32):08x})")
