"""The forward kernel's FMA-pipe exp2 (exp2_poly in csrc/sm100.cuh), replayed in float32.

The kernel evaluates 2^x for part of the softmax probabilities without the MUFU unit:
x = n + f with n = round(x) read from the mantissa after adding 1.5 * 2^23, a cubic in f,
and n added to the exponent field.  This test reads the coefficients from the CUDA source,
repeats the same float32 steps in numpy, and bounds the relative error against exact 2^x
over the range the softmax produces (x <= 0 up to the lazy-rescale slack of 8, and the
clamp at -125 for masked entries).
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "causal_sliding_window_b200", "csrc", "sm100.cuh")


def coefficients():
    text = open(SRC).read()
    body = text[text.index("float exp2_poly(float x)"):]
    vals = dict(re.findall(r"(kC[0-3]) = ([0-9.e+-]+)f", body))
    return [np.float32(vals[f"kC{i}"]) for i in range(4)]


def exp2_poly_f32(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0))).astype(np.float32)
    # fmaf(a, b, c) rounds once; in float64 then rounding to float32 reproduces it for these sizes.
    fma = lambda a, b, c: (a.astype(np.float64) * b.astype(np.float64) + np.float64(c)).astype(np.float32)  # noqa: E731
    p = fma(fma(fma(np.full_like(f, c3), f, c2), f, c1), f, c0)
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_over_softmax_range():
    x = np.concatenate([np.linspace(-125.0, 9.0, 2_000_001), -np.logspace(-8, 2, 10001)]).astype(np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1e-4          # bf16 rounding of P is 2^-9 ~ 2e-3
    assert np.all(got > 0)


def test_masked_entries_are_negligible():
    y = exp2_poly_f32(np.array([-np.inf, -1e30, -126.0], dtype=np.float32))
    assert np.all(y > 0) and np.all(y < 1e-37)


def test_exact_at_integers():
    x = np.arange(-120, 9, dtype=np.float32)
    got = exp2_poly_f32(x).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)) < 1e-4
