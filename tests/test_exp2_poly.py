"""CPU model of the FMA-pipe exp2 (ex2_poly2 in csrc/sm100.cuh), step by step in
fp32, checked against the exact 2^x.

The attention kernel evaluates one softmax exponential in four with this code
instead of the MUFU instruction; its result is rounded to bf16 (relative 2^-9)
right after, so the polynomial must stay well below that. This model uses the
coefficients read from the header, so a change there is tested here.
"""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def coefficients():
    src = open(os.path.join(ROOT, "compressive_memory_transformer_b200", "csrc", "sm100.cuh")).read()
    body = src[src.index("ex2_poly2(float a"):]
    body = body[:body.index("\n}\n")]
    c = [float(x) for x in re.findall(r"f2pack\(([0-9.]+)f, \1f\)", body)]
    # Horner order in the source: c3, c2, c1, c0
    assert len(c) == 4, c
    return np.float32(c[3]), np.float32(c[2]), np.float32(c[1]), np.float32(c[0])


def fma32(a, b, c):
    """fp32 fused multiply-add: exact product and sum, one rounding."""
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def ex2_model(x):
    c0, c1, c2, c3 = coefficients()
    k = np.float32(12582912.0)
    x = np.maximum(np.float32(x), np.float32(-126.0)).astype(np.float32)
    t = (x + k).astype(np.float32)
    n = (t - k).astype(np.float32)
    f = fma32(n, np.float32(-1.0), x)
    p = fma32(f, c3, c2)
    p = fma32(p, f, c1)
    p = fma32(p, f, c0)
    ni = t.view(np.int32) - np.array([k], dtype=np.float32).view(np.int32)[0]
    return (p.view(np.int32) + (ni << 23)).astype(np.int32).view(np.float32)


def test_relative_error_on_softmax_range():
    # arguments s*log2(e)/sqrt(d) - m are <= 8 (rescale threshold) and unbounded below
    x = np.linspace(-120.0, 8.0, 2_000_001).astype(np.float32)
    got = ex2_model(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 1.0e-4, rel.max()


def test_reduction_boundaries_and_extremes():
    for x in [-0.5, 0.5, -1.5, 1.5, 0.0, 1.0, -1.0, 7.999, -125.5]:
        got = float(ex2_model(np.array([x], np.float32))[0])
        assert abs(got / 2.0 ** x - 1) < 1e-4, x
    tiny = ex2_model(np.array([-np.inf, -1e30, -126.0, -200.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)
