"""The prefill kernel can compute part of its softmax exponentials on the FMA
pipe as 2^x = 2^round(x) * p(x - round(x)) with a cubic p on [-1/2, 1/2]
(`ex2_poly2`, packed f32x2). This checks that scheme's error bound,
evaluated step by step in fp32 with the coefficients read from the kernel
source: relative error below 1.1e-4 (well under the bf16 rounding of the
weights it feeds), exact at the integers, monotone, and 2^-125 below -125."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "pagedattention_paged_kv_02_b200", "csrc", "prefill.cuh")


def coefficients():
    body = open(SRC).read()
    fn = body[body.index("float2 ex2_poly2(float2 x)"):]
    fn = fn[:fn.index("return")]
    num = r"([-\d.e]+)f"
    c3c2 = re.search(r"__ffma2_rn\(make_float2\(" + num + r", [-\d.e]+f\), f,\s*make_float2\(" +
                     num, fn)
    c1 = re.search(r"__ffma2_rn\(p, f, make_float2\(" + num + r", [-\d.e]+f\)\);\s*p = "
                   r"__ffma2_rn\(p, f, make_float2\(1.f", fn)
    assert c3c2 and c1, "polynomial not found"
    return np.float32(c1.group(1)), np.float32(c3c2.group(2)), np.float32(c3c2.group(1))


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


def test_exact_at_integers():
    x = np.arange(-120, 9, dtype=np.float32)
    assert np.all(ex2_poly(x) == np.exp2(x))


def test_monotone_on_fine_grid():
    x = np.linspace(-20, 8, 1_000_001, dtype=np.float32)
    y = ex2_poly(x)
    assert np.all(np.diff(y) >= 0)


def test_clamped_below():
    x = np.array([-126.0, -1000.0, -3.0e38], dtype=np.float32)
    assert np.all(ex2_poly(x) == np.float32(2.0 ** -125))
