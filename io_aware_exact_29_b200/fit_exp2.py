"""Fit the cubic that the forward kernel uses for part of its 2^x evaluations.

Method: Cody & Waite range reduction x = n + f with n = round(x), f in
[-1/2, 1/2], so 2^x = 2^n * 2^f; 2^f is approximated by a cubic whose
coefficients minimise the maximum *relative* error on [-1/2, 1/2], found by
the Remez exchange algorithm (equioscillation on 5 reference points).  The
2^n factor is applied by adding n to the float's exponent field.

    python -m io_aware_exact_29_b200.fit_exp2

prints the coefficients (as written into csrc/ptx.cuh) and the error bound
that tests/test_exp2_poly.py checks.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def _solve(ref):
    # p(x_i) - 2^x_i = (-1)^i * E * 2^x_i   (relative error equioscillates)
    n = DEGREE + 2
    A = np.zeros((n, n))
    b = np.zeros(n)
    for i, x in enumerate(ref):
        A[i, :DEGREE + 1] = [x ** k for k in range(DEGREE + 1)]
        A[i, DEGREE + 1] = -((-1) ** i) * 2.0 ** x
        b[i] = 2.0 ** x
    sol = np.linalg.solve(A, b)
    return sol[:DEGREE + 1], sol[DEGREE + 1]


def rel_err(c, x):
    p = np.polyval(c[::-1], x)
    return (p - 2.0 ** x) / 2.0 ** x


def remez(iters=30):
    k = np.arange(DEGREE + 2)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (DEGREE + 1))
    grid = np.linspace(LO, HI, 200001)
    c = None
    for _ in range(iters):
        c, _ = _solve(ref)
        e = rel_err(c, grid)
        # new reference: the extremum of each sign-alternating segment
        sign = np.sign(e)
        cuts = np.flatnonzero(np.diff(sign) != 0) + 1
        segs = np.split(np.arange(grid.size), cuts)
        ext = [s[np.argmax(np.abs(e[s]))] for s in segs if s.size]
        if len(ext) < DEGREE + 2:
            break
        # keep the DEGREE+2 largest alternating extrema
        while len(ext) > DEGREE + 2:
            mags = [abs(e[i]) for i in ext]
            drop = 0 if mags[0] < mags[-1] else len(ext) - 1
            ext.pop(drop)
        ref = grid[ext]
    return c, float(np.max(np.abs(rel_err(c, grid))))


def coefficients_f32():
    c, _ = remez()
    return [float(np.float32(v)) for v in c]


if __name__ == "__main__":
    c, err = remez()
    cf = coefficients_f32()
    print("coefficients c0..c3 (fp32):", [f"{v:.9g}" for v in cf])
    print(f"max relative error of the real-valued cubic on [-1/2, 1/2]: {err:.3e}")
    grid = np.linspace(LO, HI, 200001)
    print(f"with fp32-rounded coefficients: {np.max(np.abs(rel_err(np.array(cf), grid))):.3e}")
