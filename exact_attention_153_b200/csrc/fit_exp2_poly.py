"""Fit the polynomial the attention kernel uses for part of its 2^x evaluations.

    python exact_attention_153_b200/csrc/fit_exp2_poly.py

The kernel splits x = j + f with j = round(x) (an integer, applied by adding
j to the float exponent field) and f in [-1/2, 1/2], and approximates 2^f by
a degree-3 polynomial.  This script computes its coefficients as the
minimax fit in *relative* error over [-1/2, 1/2] with the Remez exchange
algorithm (numpy only), prints them as float32 literals and reports the
error, including the float32 Horner evaluation.

Accuracy target: P is rounded to fp16 (relative step 2^-11) or bf16 (2^-8)
before the P V product, so a relative error near 1e-4 adds little; the row
sum uses the same approximated values, so the softmax weights stay
normalised.
"""
from __future__ import annotations

import numpy as np

DEGREE = 3
LO, HI = -0.5, 0.5


def remez_relative(degree: int = DEGREE, iters: int = 30):
    """Minimax polynomial p for 2^f on [LO, HI] minimising max |p/2^f - 1|."""
    n = degree + 2
    # Chebyshev extrema as the initial reference
    k = np.arange(n)
    ref = 0.5 * (LO + HI) + 0.5 * (HI - LO) * np.cos(np.pi * k[::-1] / (n - 1))
    grid = np.linspace(LO, HI, 200001)
    coef = None
    for _ in range(iters):
        # solve p(x_i) - 2^x_i = (-1)^i E 2^x_i  for coefficients and E
        A = np.zeros((n, n))
        for i, x in enumerate(ref):
            A[i, :degree + 1] = x ** np.arange(degree + 1)
            A[i, degree + 1] = -((-1) ** i) * 2.0 ** x
        sol = np.linalg.solve(A, 2.0 ** ref)
        coef = sol[:degree + 1]
        err = np.polynomial.polynomial.polyval(grid, coef) / 2.0 ** grid - 1.0
        # new reference: extrema of the error between sign changes
        sign = np.sign(err)
        idx = np.flatnonzero(np.diff(sign) != 0)
        segments = np.split(np.arange(grid.size), idx + 1)
        ext = [seg[np.argmax(np.abs(err[seg]))] for seg in segments]
        if len(ext) < n:
            break
        # keep the n consecutive extrema with the largest minimum magnitude
        best = max(range(len(ext) - n + 1), key=lambda s: min(abs(err[e]) for e in ext[s:s + n]))
        ref = grid[ext[best:best + n]]
    return coef


def horner_f32(coef32, f):
    """float32 Horner evaluation, the same order the kernel uses."""
    f = f.astype(np.float32)
    acc = np.full_like(f, coef32[-1])
    for c in coef32[-2::-1]:
        acc = (acc * f + np.float32(c)).astype(np.float32)
    return acc


def main():
    coef = remez_relative()
    coef32 = coef.astype(np.float32)
    f = np.linspace(LO, HI, 1000001)
    rel64 = np.max(np.abs(np.polynomial.polynomial.polyval(f, coef) / 2.0 ** f - 1.0))
    rel32 = np.max(np.abs(horner_f32(coef32, f).astype(np.float64) / 2.0 ** f - 1.0))
    for i, c in enumerate(coef32):
        print(f"c{i} = {float(c)!r}f  ({np.float32(c).view(np.uint32):#010x})")
    print(f"max relative error: {rel64:.3e} (exact coefficients), {rel32:.3e} (float32 Horner)")


if __name__ == "__main__":
    main()
