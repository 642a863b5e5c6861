"""The kernel's polynomial 2^x (FMA-pipe path) against numpy's exp2, on the CPU.

Reads the coefficients from the CUDA header, replays the kernel's float32
steps (clamp at -126, round-to-integer by adding 1.5 * 2^23, degree-3
Horner on the remainder, add the integer to the exponent field) and checks
the relative error over the range the softmax can produce (x <= 8 with the
lazy rescale threshold, x >= -126 before the clamp), and, for the
stale-max path (d = 64, and e4m3 operands) where x has no upper bound, that
the row acceptance rule (P sum below 2^15, or 448 for e4m3, and every
polynomial exponent below the limit read from the kernel) never accepts a
row holding a wrong or overflowing P.

These are consistency checks of a restated formula, not kernel evidence:
the GPU parity tests with planted dominant keys exercise the kernel itself.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "exact_attention_153_b200", "csrc", "sm100_ptx.cuh")


KERNEL = os.path.join(os.path.dirname(HEADER), "attn_fwd_sm100.cuh")


def poly_x_limit():
    text = open(KERNEL, encoding="utf-8").read()
    return float(re.search(r"POLY_X_LIMIT = ([0-9.]+)f", text).group(1))


def poly_pairs_d64():
    """Polynomial pairs per 16 at d = 64 and with e4m3 operands (one constant for both)."""
    text = open(KERNEL, encoding="utf-8").read()
    return int(re.search(r"exp_poly_pairs\(\) \{ return \(D == 64 \|\| FP8\) \? ([0-9]+) : 0; \}",
                         text).group(1))


def stale_sum_limits():
    """The two P-sum limits of the stale acceptance: (16-bit, e4m3)."""
    text = open(KERNEL, encoding="utf-8").read()
    m = re.search(r"tsum < \(FP8 \? ([0-9.]+)f : ([0-9.]+)f\)", text)
    return float(m.group(2)), float(m.group(1))


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


def test_relative_error_up_to_the_stale_limit():
    """Below the limit the polynomial is as accurate as on the rescale range."""
    x = np.linspace(8.0, poly_x_limit(), 1_000_001).astype(np.float32)
    y = kernel_exp2(x).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4, rel.max()


def test_exponent_add_wraps_past_128():
    """Why the stale path must bound x: from x = 128 the replay is NaN, negative or tiny."""
    x = np.array([128.2, 150.0, 200.0, 255.0, 300.0, 400.0, 450.0], dtype=np.float32)
    y = kernel_exp2(x).astype(np.float64)
    wrong = ~np.isfinite(y) | (y < 0) | (y < 1.0)
    assert wrong.all(), y


def _mufu_exp2(x):
    """ex2.approx.ftz on the MUFU: +inf from x = 128, flushed to 0 below -126."""
    with np.errstate(over="ignore"):
        y = np.exp2(x.astype(np.float64))
    y = np.where(x >= 128.0, np.inf, y)
    return np.where(x < -126.0, 0.0, y)


def _stale_row(x, use_limit=True, fp8=False):
    """Replay of the stale-max acceptance of one 128-key row (exp_row<D, *, true, FP8>)."""
    pairs = poly_pairs_d64()
    keys = np.arange(128)
    poly = (keys // 2) % 16 < pairs
    with np.errstate(invalid="ignore", over="ignore"):
        p = np.where(poly, kernel_exp2(x).astype(np.float64), _mufu_exp2(x))
    tsum = float(np.sum(p))
    xp_max = float(np.max(x[poly]))
    limit = stale_sum_limits()[1 if fp8 else 0]
    accepted = tsum < limit and (xp_max < poly_x_limit() if use_limit else True)
    return accepted, p


def _rows_with_one_big_key(rng):
    base = rng.uniform(-20.0, 0.0, size=128).astype(np.float32)
    for key in list(range(0, 8)) + list(range(32, 40)) + list(range(64, 72)) + [96, 101, 103, 10, 72]:
        for gap in (14.0, 15.0, 16.0, 40.0, 63.9, 64.0, 100.0, 127.9, 128.2, 150.0, 200.0, 300.0,
                    386.5, 450.0, 1000.0):
            x = base.copy()
            x[key] = np.float32(gap)
            yield key, gap, x


def test_stale_acceptance_never_admits_a_wrong_p():
    """Every accepted row has finite P below the fp16 range, each within the polynomial's error."""
    rng = np.random.default_rng(7)
    n = 0
    for key, gap, x in _rows_with_one_big_key(rng):
        accepted, p = _stale_row(x)
        ref = np.exp2(x.astype(np.float64))
        if accepted:
            n += 1
            assert np.all(np.isfinite(p)) and p.max() < 65504.0, (key, gap)
            rel = np.abs(p / ref - 1.0)
            assert rel.max() < 1.0e-4, (key, gap, rel.max())
        else:
            assert gap >= 15.0, (key, gap)  # rejected rows go to the row-max path
    assert n > 0


def test_stale_limits_are_the_formats_largest_values():
    """2^15 stays below fp16's largest finite 65504; 448 is e4m3's largest finite value."""
    assert stale_sum_limits() == (32768.0, 448.0)


def test_stale_acceptance_e4m3_keeps_every_p_in_range():
    """e4m3: an accepted row has every P finite and below 448 (no saturation), within the
    polynomial's error; a rejected row holds a key whose P alone is at least 448 / 128."""
    rng = np.random.default_rng(11)
    n = 0
    for key, gap, x in _rows_with_one_big_key(rng):
        for g in (gap, gap - 13.0, 8.0, 8.7, 8.9):
            x2 = x.copy()
            x2[key] = np.float32(g)
            accepted, p = _stale_row(x2, fp8=True)
            if accepted:
                n += 1
                ref = np.exp2(x2.astype(np.float64))
                assert np.all(np.isfinite(p)) and p.max() < 448.0, (key, g)
                assert np.abs(p / ref - 1.0).max() < 1.0e-4, (key, g)
            else:
                assert g > np.log2(448.0 / 128.0), (key, g)
    assert n > 0


def test_sum_check_alone_would_admit_wrapped_values():
    """Without the exponent limit a dominant key in a polynomial slot passes the sum check."""
    x = np.full(128, -3.0, dtype=np.float32)
    x[3] = np.float32(150.0)  # key 3: pair 1, a polynomial slot
    accepted_without_limit, p = _stale_row(x, use_limit=False)
    assert accepted_without_limit and p[3] < 1.0  # the silent wrong answer
    accepted, _ = _stale_row(x)
    assert not accepted
