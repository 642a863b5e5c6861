"""Pins of the FP8 (e4m3) oracle, each against something other than the oracle itself.

* The e4m3 decoder against the format's definition (hand-computed values of
  named codes), against torch's own float8_e4m3fn conversion on all 256
  codes, and against the ordering every sign-magnitude float has.
* The dequantised attention against the pure-Python brute force (shares no
  arithmetic), torch's float64 scaled_dot_product_attention, and the closed
  form of a single visible key.
* The V transposition against index-by-index reading on a shape with
  Nk != d, so a transposed operand cannot pass.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention_fp8_f64, brute_force, decode_e4m3, dequantize_e4m3, untranspose_v
from seeded_inputs import make_fp8_qkv

ALL_CODES = np.arange(256, dtype=np.uint8)


def test_named_codes_from_the_definition():
    # (code, value) written out from sign / exponent (bias 7) / mantissa fields
    cases = [(0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6),
             (0x38, 1.0), (0x3C, 1.5), (0x40, 2.0), (0x7E, 448.0), (0x77, 240.0),
             (0xB8, -1.0), (0xFE, -448.0), (0x81, -(2.0 ** -9))]
    got = decode_e4m3(np.array([c for c, _ in cases], dtype=np.uint8))
    assert got.tolist() == [v for _, v in cases]
    assert np.isnan(decode_e4m3(np.array([0x7F, 0xFF], dtype=np.uint8))).all()
    assert math.copysign(1.0, decode_e4m3(np.array([0x80], dtype=np.uint8))[0]) == -1.0


def test_all_codes_match_torch_float8():
    ref = torch.from_numpy(ALL_CODES.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = decode_e4m3(ALL_CODES)
    nan = np.isnan(ref)
    assert (np.isnan(ours) == nan).all()
    assert (ours[~nan] == ref[~nan]).all()


def test_codes_are_ordered_like_sign_magnitude():
    pos = decode_e4m3(ALL_CODES[:127])  # 0x00 .. 0x7E
    assert (np.diff(pos) > 0).all()
    neg = decode_e4m3(ALL_CODES[128:255])
    assert (neg == -pos).all()


def test_decode_accepts_torch_tensors():
    t = torch.tensor([1.0, -0.5, 448.0, 2.0 ** -9], dtype=torch.float32).to(torch.float8_e4m3fn)
    assert decode_e4m3(t).tolist() == [1.0, -0.5, 448.0, 2.0 ** -9]


def test_dequantize_scales_every_value():
    assert dequantize_e4m3(np.array([0x38, 0x7E], dtype=np.uint8), 0.25).tolist() == [0.25, 112.0]


def test_untranspose_reads_index_by_index():
    rng = np.random.default_rng(0)
    vt = rng.standard_normal((2, 3, 4, 7))  # [B, H, d, Nk] with Nk != d
    v = untranspose_v(vt)
    assert v.shape == (2, 3, 7, 4)
    for b, h, j, c in np.ndindex(*v.shape):
        assert v[b, h, j, c] == vt[b, h, c, j]


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_brute_force(causal):
    q8, k8, vt8, (qs, ks, vs) = make_fp8_qkv(1, 2, 5, 6, 8, seed=11)
    o, lse = attention_fp8_f64(q8, k8, vt8, qs, ks, vs, scale=0.35, causal=causal)
    q = torch.from_numpy(decode_e4m3(q8) * qs)
    k = torch.from_numpy(decode_e4m3(k8) * ks)
    v = torch.from_numpy(decode_e4m3(vt8) * vs).transpose(-1, -2)
    bo, bl = brute_force(q, k, v, 0.35, causal)
    np.testing.assert_allclose(o, np.array(bo), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, np.array(bl), rtol=0, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_attention_matches_torch_sdpa_float64(causal):
    q8, k8, vt8, (qs, ks, vs) = make_fp8_qkv(2, 2, 37, 37, 128, seed=5)
    o, _ = attention_fp8_f64(q8, k8, vt8, qs, ks, vs, causal=causal)
    q = q8.to(torch.float64) * qs
    k = k8.to(torch.float64) * ks
    v = (vt8.to(torch.float64) * vs).transpose(-1, -2)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def test_single_key_returns_its_value_row():
    q8, k8, vt8, (qs, ks, vs) = make_fp8_qkv(1, 1, 3, 1, 16, seed=2)
    o, lse = attention_fp8_f64(q8, k8, vt8, qs, ks, vs)
    v_row = decode_e4m3(vt8)[0, 0, :, 0] * vs
    for i in range(3):
        assert (o[0, 0, i] == v_row).all()
    s = (decode_e4m3(q8)[0, 0] * qs) @ (decode_e4m3(k8)[0, 0, 0] * ks) / 4.0
    np.testing.assert_allclose(lse[0, 0], s, rtol=0, atol=1e-14)


def test_generator_puts_each_tensors_peak_on_448():
    q8, k8, vt8, scales = make_fp8_qkv(1, 2, 64, 48, 128, seed=9)
    for t in (q8, k8, vt8):
        assert float(t.to(torch.float32).abs().max()) == 448.0
    assert vt8.shape == (1, 2, 128, 48)
    assert all(s > 0 for s in scales)


# --- planted mistakes: each must make at least one pin above fail ------------------------

_decode = decode_e4m3  # the true decoder, which the mutants below start from


def _decode_bias8(codes):
    return _decode(codes) / 2.0


def _decode_no_subnormals(codes):
    c = codes.view(torch.uint8).numpy() if hasattr(codes, "detach") else np.asarray(codes)
    e = (c.astype(np.int64) >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    return np.where(e == 0, sign * (1.0 + m / 8.0) * 2.0 ** -7, _decode(c))


def _decode_unsigned(codes):
    return np.abs(_decode(codes))


def _untranspose_identity(vt):
    return np.ascontiguousarray(vt)


def _untranspose_reshape(vt):
    return np.ascontiguousarray(vt).reshape(*vt.shape[:-2], vt.shape[-1], vt.shape[-2])


def _pins():
    return [test_named_codes_from_the_definition, test_all_codes_match_torch_float8,
            test_codes_are_ordered_like_sign_magnitude, test_decode_accepts_torch_tensors,
            test_dequantize_scales_every_value, test_untranspose_reads_index_by_index,
            lambda: test_attention_matches_brute_force(False),
            lambda: test_attention_matches_torch_sdpa_float64(True),
            test_single_key_returns_its_value_row]


@pytest.mark.parametrize("name,mutant", [("decode_e4m3", _decode_bias8),
                                         ("decode_e4m3", _decode_no_subnormals),
                                         ("decode_e4m3", _decode_unsigned),
                                         ("untranspose_v", _untranspose_identity),
                                         ("untranspose_v", _untranspose_reshape)])
def test_pins_catch_planted_mistakes(monkeypatch, name, mutant):
    """The mutant replaces the oracle function everywhere the pins reach it."""
    import oracle.fp8 as F
    monkeypatch.setattr(F, name, mutant)
    monkeypatch.setitem(globals(), name, mutant)
    failed = 0
    for pin in _pins():
        try:
            pin()
        except (AssertionError, ValueError):  # a pin that raises has failed too
            failed += 1
    assert failed > 0
