"""The FP8 forward's FMA-pipe 2^x (csrc/fa_device.cuh, exp2_poly_x2): its coefficients and its
range reduction, checked on the CPU against the exact 2^x.

The kernel rounds P to e4m3 (3 mantissa bits, relative step 2^-4), so the polynomial only has
to stay far inside that; the header states a maximum relative error of 7.5e-5.  These tests
read the four coefficients from the header and check that bound (fp64 Horner on [-1/2, 1/2]),
then replay the kernel's fp32 steps (n = round(x) by adding and subtracting 1.5 * 2^23, Horner
in fp32, n added to the exponent field) over the inputs the kernel feeds it (x in [-125, 0]).
"""
import os
import re

import numpy as np
import pytest

HDR = os.path.join(os.path.dirname(__file__), "..", "exact_io_aware_97_b200", "csrc", "fa_device.cuh")


def _coeffs():
    src = open(HDR).read()
    vals = {}
    for i in range(4):
        m = re.search(rf"constexpr float kExp2C{i} = ([0-9.eE+-]+)f;", src)
        assert m, f"kExp2C{i} not found"
        vals[i] = float(m.group(1))
    return [vals[i] for i in range(4)]


def test_poly_relative_error_on_reduced_range():
    c0, c1, c2, c3 = _coeffs()
    f = np.linspace(-0.5, 0.5, 200001)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= 7.6e-5, rel.max()
    # equioscillation of a minimax fit: the error reaches its bound at both ends and inside
    assert rel[0] > 0.5 * rel.max() and rel[-1] > 0.5 * rel.max()


def _kernel_exp2(x):
    """The kernel's steps in fp32 (packed FMA ops evaluated one lane at a time)."""
    c0, c1, c2, c3 = (np.float32(c) for c in _coeffs())
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + magic).astype(np.float32)
    nf = (t - magic).astype(np.float32)
    fr = (x - nf).astype(np.float32)
    # fma(a, b, c) with one rounding: exact product in fp64, then round to fp32
    fma = lambda a, b, c: (a.astype(np.float64) * b + c).astype(np.float32)
    q = fma(fr, np.full_like(fr, c3), np.full_like(fr, c2))
    q = fma(q, fr, np.full_like(fr, c1))
    q = fma(q, fr, np.full_like(fr, c0))
    bits = q.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.astype(np.uint32).view(np.float32), fr


@pytest.mark.parametrize("lo,hi", [(-125.0, -100.0), (-30.0, -1.0), (-1.0, 0.0)])
def test_kernel_steps_match_exp2(lo, hi):
    x = np.linspace(lo, hi, 100003, dtype=np.float32)
    y, fr = _kernel_exp2(x)
    assert np.all(np.abs(fr) <= 0.5)  # round-to-nearest reduction
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    # the fit's 7.5e-5 plus a few fp32 roundings
    assert rel.max() <= 8e-5, rel.max()


def test_inputs_below_range_clamp():
    y, _ = _kernel_exp2(np.array([-200.0, -126.0, -np.inf], dtype=np.float32))
    assert np.allclose(y.astype(np.float64), 2.0 ** -125, rtol=1e-4)
