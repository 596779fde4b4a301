"""The forward kernel's FMA-pipe 2^x (ptx.cuh, exp2_poly2) against exact 2^x.

The kernel evaluates a quarter of its softmax exponentials with a Cody &
Waite range reduction and a minimax cubic.  This emulates the same fp32
operation sequence in numpy and checks the error bound over the whole input
range the kernel can produce (x <= 8 with lazy rescaling, down to -inf), and
that the coefficients in the CUDA source are the ones the fit produces.
"""
import os
import re

import numpy as np

from io_aware_exact_29_b200 import fit_exp2

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "io_aware_exact_29_b200", "csrc", "ptx.cuh")


def _source_constants():
    with open(SRC) as fh:
        text = fh.read()
    body = text[text.index("exp2_poly2"):]
    vals = dict(re.findall(r"(kC[0-3]) = ([0-9.e+-]+)f", body))
    rnd = float(re.search(r"kRound = ([0-9.]+)f", body).group(1))
    return [np.float32(float(vals[f"kC{i}"])) for i in range(4)], np.float32(rnd)


def _emulate(x):
    """fp32 emulation of exp2_poly2 on a vector."""
    (c0, c1, c2, c3), rnd = _source_constants()
    f32 = np.float32
    xc = np.maximum(x.astype(f32), f32(-127.0))
    rr = (xc + rnd).astype(f32)
    fr = (xc - (rr - rnd).astype(f32)).astype(f32)
    q = (fr * c3 + c2).astype(f32)   # fma rounding differs by <= 1 ulp per step
    q = (q * fr + c1).astype(f32)
    q = (q * fr + c0).astype(f32)
    scale = (rr.view(np.int32) << 23).view(f32)
    return (q * scale).astype(f32)


def test_source_coefficients_are_the_fit():
    (c0, c1, c2, c3), rnd = _source_constants()
    fit = fit_exp2.coefficients_f32()
    assert [float(c) for c in (c0, c1, c2, c3)] == [float(np.float32(v)) for v in fit]
    assert float(rnd) == 1.5 * 2 ** 23 + 127


def test_relative_error_bound_over_the_kernel_range():
    x = np.concatenate([np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64),
                        np.arange(-126, 9, dtype=np.float64) + 0.5,
                        np.arange(-126, 9, dtype=np.float64)])
    x = x.astype(np.float32)
    got = _emulate(x).astype(np.float64)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got - exact) / exact
    # 7.48e-5 from the cubic plus a few fp32 roundings in the evaluation
    assert rel.max() < 7.5e-5 + 8 * 2.0 ** -24, rel.max()


def test_underflow_and_minus_infinity_are_exact_zero():
    x = np.array([-np.inf, -1e30, -200.0, -127.0, -127.4], dtype=np.float32)
    assert np.all(_emulate(x) == 0.0)
    # just above the clamp the value is normal and accurate
    v = _emulate(np.array([-126.0], dtype=np.float32))[0]
    assert abs(float(v) / 2.0 ** -126 - 1.0) < 1e-4
