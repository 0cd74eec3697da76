"""CPU check of the polynomial exp2 used for part of the softmax
exponentials in the tensor-core kernel (csrc/exp2_poly.h): the same steps in
float32 / int32 arithmetic (round-to-nearest magic-number reduction, degree-3
Horner, exponent-field add) stay within the stated relative-error bound of
2^x over the range the kernel feeds it."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "causal_attention_rtr_b200", "csrc", "exp2_poly.h")


def coefficients():
    text = open(HDR).read()
    return [np.float32(float(re.search(r"#define RTR_EXP2_C%d ([0-9.eE+-]+)f" % i, text).group(1)))
            for i in range(4)]


def exp2_poly_emulated(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = (x - n).astype(np.float32)
    # fmaf: single rounding of a*b+c; float64 holds the exact product of two
    # float32 values, so rounding a*b+c once to float32 reproduces it.
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)
    p = fma(np.full_like(f, c3), f, c2)
    p = fma(p, f, c1)
    p = fma(p, f, c0)
    bits = p.view(np.int32) + (t.view(np.int32) << np.int32(23))
    return bits.view(np.float32)


def test_reduction_range():
    x = np.linspace(-40, 10, 100001).astype(np.float32)
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    f = (x - (t - magic).astype(np.float32)).astype(np.float32)
    assert np.all(np.abs(f) <= 0.5)


def test_relative_error_bound():
    x = np.concatenate([np.linspace(-120, 10, 2_000_001), np.array([0.0, -1.0, 0.5, -0.5, 8.0, -8.0])])
    x = x.astype(np.float32)
    got = exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 8e-5, rel.max()


def test_clamp_is_tiny_and_positive():
    got = exp2_poly_emulated(np.array([-125.0, -200.0, -1e30], np.float32))
    assert np.all(got > 0) and np.all(got < 2.0 ** -120)
