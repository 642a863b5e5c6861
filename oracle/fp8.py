"""Float64 CPU oracle for the FP8 (e4m3) attention forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
CUDA product path never calls it and shares no code with it.

What it computes.  "一个反直觉的事实：大模型推理的瓶颈不是计算，而是显存"
(ai2ai.xin), section "FlashAttention-3的进一步增强", item 2, says only that
FlashAttention-3 runs the attention in FP8 at half the memory.  Read plainly:
the inputs arrive as 8-bit floating-point codes with one scale factor per
tensor, and the method computes the same exact attention as before on the
values those codes stand for.  So the oracle

* decodes every e4m3 code from the format's definition (below),
* multiplies by the tensor's descale factor (value = decode(code) * descale),
* takes V from its transposed [B, H, d, Nk] layout back to [B, H, Nk, d],
* and runs the float64 definition of attention on the result
  (``oracle.attention.attention_f64``).

The e4m3 format (the OCP 8-bit floating point definition, "E4M3"): bit 7 is
the sign, bits 6..3 the exponent e with bias 7, bits 2..0 the mantissa m.
e = 0 encodes the subnormals (m / 8) * 2^-6; e = 1..15 encode
(1 + m / 8) * 2^(e - 7), except e = 15 with m = 7, which is NaN.  There are
no infinities; the largest finite magnitude is 1.75 * 2^8 = 448.

Every function is pinned by ``tests/test_oracle_fp8.py``.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_f64, to_f64

__all__ = ["decode_e4m3", "dequantize_e4m3", "untranspose_v", "attention_fp8_f64"]


def _codes(x) -> np.ndarray:
    """The raw 8-bit codes of a uint8 array, or of a torch float8 / uint8 tensor."""
    if hasattr(x, "detach"):
        import torch
        t = x.detach().to("cpu").contiguous()
        if t.dtype != torch.uint8:
            t = t.view(torch.uint8)
        return t.numpy()
    a = np.asarray(x)
    if a.dtype != np.uint8:
        raise TypeError("e4m3 codes must be uint8")
    return a


def decode_e4m3(codes) -> np.ndarray:
    """Float64 value of every e4m3 code (NaN for the two NaN codes)."""
    c = _codes(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (c & 0x7 == 7), np.nan, val)


def dequantize_e4m3(codes, descale: float) -> np.ndarray:
    """decode(code) * descale: the real value a scaled e4m3 tensor stands for."""
    return decode_e4m3(codes) * float(descale)


def untranspose_v(vt: np.ndarray) -> np.ndarray:
    """V [B, H, Nk, d] from its transposed layout Vt [B, H, d, Nk]."""
    return np.ascontiguousarray(np.swapaxes(vt, -1, -2))


def attention_fp8_f64(q_codes, k_codes, vt_codes, q_descale: float, k_descale: float,
                      v_descale: float, scale: float | None = None, causal: bool = False):
    """Exact attention of the dequantised inputs, in float64.

    q_codes [B, H, Nq, d], k_codes [B, H, Nk, d], vt_codes [B, H, d, Nk]: e4m3
    codes; the descales turn codes into values.  Returns (O [B, H, Nq, d],
    lse [B, H, Nq]) of softmax(scale * Q K^T) V with scale = 1 / sqrt(d) by
    default.
    """
    q = dequantize_e4m3(q_codes, q_descale)
    k = dequantize_e4m3(k_codes, k_descale)
    v = untranspose_v(dequantize_e4m3(vt_codes, v_descale))
    return attention_f64(to_f64(q), to_f64(k), to_f64(v), scale=scale, causal=causal)
