"""GPU parity of the attention block (attn_qkv_proj, attn_fwd, attn_out_proj, attn_block_fwd)
against the float64 block oracle, stage by stage and element by element.

Each stage is compared with the oracle applied to the exact inputs the GPU stage received:
the qkv projection with x and W_qkv, the attention with the GPU's q, k, v (the forward's
tolerances: 4e-3 fp16, 2e-2 bf16, lse 1e-3), the output projection with the GPU's o.  A
projection element y = sum_k a_k w_k + b is computed from exact 16-bit products with fp32
accumulation over K = C terms, the bias added in fp32 and one rounding to the dtype, so it
must lie within

    2 * (u |y| + (K + 1) 2^-24 (sum_k |a_k w_k| + |b|)) + 2^-24 max|y|

of the oracle (u = 2^-11 fp16, 2^-8 bf16; the factor 2 covers second-order terms).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
import oracle
from exact_attention_153_b200 import build_lib
from seeded_inputs import make_block_inputs

pytestmark = pytest.mark.gpu

UNIT = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}
TOL = {"fp16": 4e-3, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _f64(t):
    return t.detach().cpu().double().numpy() if t is not None else None


def _linear_ratio(got, a, w, b, u):
    """max |got - ref| / bound for y = a W^T + b (arrays in float64), and the reference."""
    ref = oracle.linear(a, w, b)
    K = a.shape[-1]
    mag = np.abs(a) @ np.abs(w).T + (np.abs(b) if b is not None else 0.0)
    tol = 2 * (u * np.abs(ref) + (K + 1) * 2.0 ** -24 * mag) + 2.0 ** -24 * np.max(np.abs(ref))
    return float(np.max(np.abs(got - ref) / tol))


CASES = [
    # B, N, H, d, C_out, dtype, causal, qkv_bias
    (1, 400, 2, 64, 128, "fp16", False, False),   # the 20x20 YOLO shape, C = 128
    (2, 100, 3, 64, 200, "bf16", False, True),    # 3C = 576 and C_out = 200: ragged column tiles
    (1, 300, 2, 128, 256, "bf16", True, False),   # d = 128
    (2, 257, 2, 64, 128, "fp16", True, True),     # ragged rows across the batch boundary
    (16, 1600, 4, 64, 256, "fp16", False, False), # the 40x40, batch 16 YOLO shape, C = 256
]


@pytest.mark.parametrize("B,N,H,d,C_out,dtype,causal,qkv_bias", CASES)
def test_block_stages_match_oracle(B, N, H, d, C_out, dtype, causal, qkv_bias):
    u = UNIT[dtype]
    x, w_qkv, b_qkv, w_o, b_o = make_block_inputs(B, N, H, d, C_out, dtype, seed=B * N + H + d,
                                                  qkv_bias=qkv_bias)
    dev = lambda t: t.cuda() if t is not None else None
    scale = 1.0 / math.sqrt(d)
    y, q, k, v, o, lse = A.block_forward(dev(x), dev(w_qkv), dev(b_qkv), dev(w_o), dev(b_o), H,
                                         causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, word = A.attn_get_device_status()
    assert st == 0, f"device status {word:#x}"
    # 1. qkv projection, every element, through the oracle's split
    C = H * d
    qkv_got = np.concatenate([oracle.merge_heads(_f64(t)) for t in (q, k, v)], axis=-1)
    r = _linear_ratio(qkv_got, _f64(x), _f64(w_qkv), _f64(b_qkv), u)
    assert r <= 1.0, f"qkv err/tol {r:.3f}"
    qr, kr, vr = oracle.split_qkv(oracle.linear(_f64(x), _f64(w_qkv), _f64(b_qkv)), H, d)
    assert np.max(np.abs(_f64(q) - qr)) <= 4 * u * max(1.0, np.max(np.abs(qr)))
    # 2. attention on the GPU's own q, k, v
    o_ref, lse_ref = oracle.attention_f64(q.cpu(), k.cpu(), v.cpu(), scale, causal)
    assert np.max(np.abs(_f64(o) - o_ref)) <= TOL[dtype]
    assert np.max(np.abs(_f64(lse) - lse_ref)) <= 1e-3
    # 3. output projection on the GPU's own o
    r = _linear_ratio(_f64(y), oracle.merge_heads(_f64(o)), _f64(w_o), _f64(b_o), u)
    assert r <= 1.0, f"proj err/tol {r:.3f}"
    print(f"\nBLOCK PARITY B={B} N={N} H={H} d={d} C_out={C_out} {dtype}: ok")


def test_separate_calls_equal_the_block_call():
    B, N, H, d, C_out = 2, 333, 2, 64, 128
    x, w_qkv, b_qkv, w_o, b_o = (t.cuda() if t is not None else None
                                 for t in make_block_inputs(B, N, H, d, C_out, "fp16", seed=5))
    y, q, k, v, o, lse = A.block_forward(x, w_qkv, b_qkv, w_o, b_o, H)
    q2, k2, v2 = A.qkv_proj(x, w_qkv, b_qkv, H)
    o2, _ = A.forward(q2, k2, v2)
    y2 = A.out_proj(o2, w_o, b_o)
    torch.cuda.synchronize()
    assert torch.equal(q, q2) and torch.equal(k, k2) and torch.equal(v, v2)
    assert torch.equal(o, o2) and torch.equal(y, y2)
