"""Coefficients of the software exp2 used by the prefill softmax.

Method: Cody-Waite style range reduction, x = j + f with j = rint(x) and
f in [-1/2, 1/2], so 2^x = 2^j * 2^f; 2^f is approximated by the degree-3
polynomial p(f) = c0 + c1 f + c2 f^2 + c3 f^3 whose maximum relative error
on [-1/2, 1/2] is minimal (minimax), found with the Remez exchange algorithm
below.  The coefficients are then rounded to float32, and the error of the
rounded polynomial, evaluated the way the kernel does it (Horner with fused
multiply-adds in float32), is measured on a dense grid.

    python -m ring_sliding_window_b200.csrc.gen_exp2_poly

prints the float32 coefficients (as C hex-float literals) and the measured
maximum relative error; the kernel's constants must equal them, which
tests/test_exp2_poly.py checks.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _remez(degree: int = DEGREE, iters: int = 40):
    n = degree
    # reference: n + 2 Chebyshev extrema on [LO, HI]
    k = np.arange(n + 2)
    xs = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * (n + 1 - k) / (n + 1))
    grid = np.linspace(LO, HI, 200_001)
    coef = None
    for _ in range(iters):
        # p(x_i) - (-1)^i E 2^{x_i} = 2^{x_i}   (equioscillating relative error E)
        A = np.zeros((n + 2, n + 2))
        for i, x in enumerate(xs):
            A[i, :n + 1] = x ** np.arange(n + 1)
            A[i, n + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** xs)
        coef = sol[:n + 1]
        err = np.polyval(coef[::-1], grid) / 2.0 ** grid - 1.0
        # new reference: the extremum of each sign-alternating run of the error
        sign = np.sign(err)
        sign[sign == 0] = 1
        cuts = np.nonzero(np.diff(sign))[0] + 1
        runs = np.split(np.arange(grid.size), cuts)
        ext = [r[np.argmax(np.abs(err[r]))] for r in runs]
        if len(ext) < n + 2:
            break
        # keep n + 2 alternating extrema with the largest errors
        while len(ext) > n + 2:
            if abs(err[ext[0]]) < abs(err[ext[-1]]):
                ext = ext[1:]
            else:
                ext = ext[:-1]
        new_xs = grid[ext]
        if np.allclose(new_xs, xs, atol=1e-12):
            break
        xs = new_xs
    return coef


def _fma32(a, b, c):
    """float32 fused multiply-add: exact product and sum in float64, one rounding."""
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def eval_kernel_order(c32, x32):
    """p(x) in float32 with the kernel's Horner/FMA order (vectorised)."""
    a = np.float64(c32[3]) * x32.astype(np.float64) + np.float64(c32[2])
    a = a.astype(np.float32)
    a = (a.astype(np.float64) * x32 + np.float64(c32[1])).astype(np.float32)
    a = (a.astype(np.float64) * x32 + np.float64(c32[0])).astype(np.float32)
    return a


def coefficients():
    """(float32 coefficients c0..c3, measured max relative error of p on [-1/2, 1/2])."""
    c = _remez()
    c32 = np.array(c, dtype=np.float32)
    x = np.linspace(LO, HI, 1_000_001).astype(np.float32)
    rel = np.abs(eval_kernel_order(c32, x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1)
    return c32, float(rel.max())


def main():
    c32, err = coefficients()
    for i, v in enumerate(c32):
        print(f"c{i} = {float(v).hex()}f  // {float(v):.9g}")
    print(f"max relative error on [-1/2, 1/2] (float32 Horner): {err:.3e}")


if __name__ == "__main__":
    main()
