"""The prefill kernel computes part of its softmax exponentials as
2^x = 2^round(x) * p(x - round(x)) with a cubic p on [-1/2, 1/2]. This checks
the claimed error bound of that scheme, evaluated step by step in fp32 with
the coefficients read from the kernel source: relative error below 1.1e-4
(well under the bf16 rounding of the weights), exact at 0, monotone."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "pagedattention_paged_kv_02_b200", "csrc", "prefill.cuh")


def coefficients():
    body = open(SRC).read()
    fn = body[body.index("float ex2_poly(float x)"):]
    fn = fn[:fn.index("}")]
    c = re.findall(r"fmaf\(fmaf\(fmaf\(([-\d.e]+)f, f, ([-\d.e]+)f\), f, ([-\d.e]+)f\), f, 1.f\)",
                   fn)
    assert c, "polynomial not found"
    c3, c2, c1 = (np.float32(v) for v in c[0])
    return c1, c2, c3


def ex2_poly(x):
    c1, c2, c3 = coefficients()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125))
    t = (x + f32(12582912.0)).astype(f32)
    n = (t - f32(12582912.0)).astype(f32)
    fr = (x - n).astype(f32)
    p = ((c3 * fr + c2).astype(f32) * fr + c1).astype(f32)
    p = (p * fr + f32(1)).astype(f32)
    return (p.view(np.int32) + (t.view(np.int32) << 23)).view(f32)


def test_relative_error_bound():
    x = np.linspace(-100, 8, 4_000_001, dtype=np.float32)
    got = ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 1.1e-4


def test_exact_at_integers_and_zero():
    x = np.arange(-120, 9, dtype=np.float32)
    assert np.all(ex2_poly(x) == np.exp2(x))


def test_monotone_on_fine_grid():
    x = np.linspace(-20, 8, 1_000_001, dtype=np.float32)
    y = ex2_poly(x)
    assert np.all(np.diff(y) >= 0)
