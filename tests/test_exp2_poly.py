"""The kernel's polynomial 2^x (FMA-pipe path) against numpy's exp2, on the CPU.

Reads the coefficients from the CUDA header, replays the kernel's float32
steps (clamp at -126, round-to-integer by adding 1.5 * 2^23, degree-3
Horner on the remainder, add the integer to the exponent field) and checks
the relative error over the range the softmax can produce (x <= 8 with the
lazy rescale threshold, x >= -126 before the clamp).
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "exact_attention_153_b200", "csrc", "sm100_ptx.cuh")


def coefficients():
    text = open(HEADER, encoding="utf-8").read()
    body = text[text.index("void exp2_poly2"):]
    vals = dict(re.findall(r"\b(c[0-3]) = ([0-9.eE+-]+)f", body))
    return [np.float32(float(vals[f"c{i}"])) for i in range(4)]


def kernel_exp2(x):
    c = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-126.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    j = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (c[3] * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_in_range():
    x = np.linspace(-120.0, 8.5, 2_000_001).astype(np.float32)
    y = kernel_exp2(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.0e-4, rel.max()


def test_integers_and_halves():
    x = np.arange(-100, 9, dtype=np.float32)
    assert np.max(np.abs(kernel_exp2(x) / np.exp2(x.astype(np.float64)) - 1)) < 1e-4
    x = x + np.float32(0.5)
    assert np.max(np.abs(kernel_exp2(x) / np.exp2(x.astype(np.float64)) - 1)) < 1e-4


def test_masked_inputs_give_tiny_nonnegative_values():
    x = np.array([-np.inf, -1e30, -500.0, -126.0, -125.9], dtype=np.float32)
    y = kernel_exp2(x)
    assert np.all(y >= 0) and np.all(np.isfinite(y)) and np.all(y < 2.0 ** -125)


def test_monotone_on_a_fine_grid():
    x = np.linspace(-30.0, 8.0, 400_001).astype(np.float32)
    y = kernel_exp2(x)
    # the polynomial is not exactly monotone across integer splits, but any
    # step down is far below the fp16 rounding of P
    d = np.diff(y.astype(np.float64)) / y[:-1]
    assert d.min() > -2e-4
