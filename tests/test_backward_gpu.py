"""GPU parity of the backward (attn_bwd) against the float64 backward oracle.

Two comparisons per case, both element by element over dQ, dK and dV:

1. Kernel parity: the oracle applied to exactly the inputs the kernel gets --
   q, k, v, dO and the forward's saved o and lse as the GPU produced them.
   The kernel's own arithmetic differs from that only by rounding: P is
   recomputed in fp32 and rounded to the input dtype for dV = P^T dO; dS is
   formed in fp32 from that rounded P and rounded for dK = dS^T Q and
   dQ = dS K; the tensor core accumulates in fp32; the results are rounded
   once.  With u the unit roundoff of the dtype (2^-11 fp16, 2^-8 bf16), each
   element must therefore lie within

       2 * (2u * sum_i |a_i b_i| + u * |result|) + floor

   of the oracle, where sum_i |a_i b_i| is the product of the absolute values
   of the two operands of that element's contraction (|P|^T |dO| for dV,
   scale |dS| |K| for dQ, scale |dS|^T |Q| for dK): one rounding of the
   operand that is rounded, one of the result, a factor 2 for second-order
   terms, and a floor of 2^-20 * max|result| for the fp32 accumulation.
   dS = P (dP - D) subtracts two fp32 dot products that can cancel, so the
   dQ and dK bounds also carry 2^-22 P (|dO| |V|^T + rowsum(|dO| |o|)), the
   fp32 rounding of dP and D, through their contraction.
2. End to end: forward then backward against the exact gradient (the oracle's
   own float64 forward).  The bound adds the propagation of the forward's
   error in o and lse: dS changes by P * |delta D| + |dS| * |delta lse| with
   delta D = rowsum(dO * (o_gpu - o_exact)), and P by P * |delta lse|.
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
import oracle
from exact_attention_153_b200 import build_lib
from oracle.backward import recompute_probs, grad_p, row_dot, grad_scores
from oracle.attention import apply_causal_mask, scores
from seeded_inputs import WORKLOADS, make_grad_out, make_qkv, make_workload_qkv

pytestmark = pytest.mark.gpu

UNIT = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _f64(t):
    return t.detach().cpu().double().numpy()


def _gpu_forward_backward(q, k, v, do, causal, scale):
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = A.forward(qd, kd, vd, causal=causal, scale=scale)
    dq, dk, dv = A.backward(qd, kd, vd, o, lse, dod, causal=causal, scale=scale)
    torch.cuda.synchronize()
    st, word = A.attn_get_device_status()
    assert st == 0, f"device status {word:#x}"
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def _bounds(q, k, v, do, o, lse, scale, causal, u, o_exact=None, lse_exact=None):
    """Per-element bounds for dQ, dK, dV of one (batch, head) (arrays in float64).

    With o_exact / lse_exact, the bound also covers the difference between
    the saved statistics (o, lse) and the exact forward's.
    """
    rows = np.arange(q.shape[0])
    s = scores(q, k, scale)
    if causal:
        s = apply_causal_mask(s, rows)
    p = recompute_probs(s, lse)
    dp = grad_p(do, v)
    ds = grad_scores(p, dp, row_dot(do, o))
    ap, ads = np.abs(p), np.abs(ds)
    # fp32 rounding of dP and D, which dS = P (dP - D) subtracts
    e32 = 2.0 ** -22 * ap * (np.abs(do) @ np.abs(v).T + row_dot(np.abs(do), np.abs(o))[:, None])
    b_dv = 2 * u * (ap.T @ np.abs(do))
    b_dq = scale * (2 * u * (ads @ np.abs(k)) + e32 @ np.abs(k))
    b_dk = scale * (2 * u * (ads.T @ np.abs(q)) + e32.T @ np.abs(q))
    if o_exact is not None:
        dlse = np.abs(lse - lse_exact)
        dD = np.abs(row_dot(do, o - o_exact))
        e_ds = ap * dD[:, None] + ads * dlse[:, None]
        b_dv = b_dv + (ap * dlse[:, None]).T @ np.abs(do)
        b_dq = b_dq + scale * (e_ds @ np.abs(k))
        b_dk = b_dk + scale * (e_ds.T @ np.abs(q))
    return b_dq, b_dk, b_dv


def _check(q, k, v, do, causal, scale, dtype, end_to_end=True):
    u = UNIT[dtype]
    o, lse, dq, dk, dv = _gpu_forward_backward(q, k, v, do, causal, scale)
    # 1. kernel parity: the oracle on the same saved statistics
    ref = oracle.attention_backward_f64(q, k, v, do, scale, causal, o=o, lse=lse)
    if end_to_end:
        exact = oracle.attention_backward_f64(q, k, v, do, scale, causal)
        o_ex, lse_ex = oracle.attention_f64(q, k, v, scale, causal)
    qf, kf, vf, dof, of, lf = _f64(q), _f64(k), _f64(v), _f64(do), _f64(o), _f64(lse)
    worst = {}
    B, H = q.shape[0], q.shape[1]
    for name, got in (("dq", dq), ("dk", dk), ("dv", dv)):
        worst[name] = 0.0
    for b in range(B):
        for h in range(H):
            bounds = _bounds(qf[b, h], kf[b, h], vf[b, h], dof[b, h], of[b, h], lf[b, h], scale,
                             causal, u)
            if end_to_end:
                bounds_e2e = _bounds(qf[b, h], kf[b, h], vf[b, h], dof[b, h], of[b, h], lf[b, h],
                                     scale, causal, u, o_ex[b, h], lse_ex[b, h])
            for idx, (name, got) in enumerate((("dq", dq), ("dk", dk), ("dv", dv))):
                g = _f64(got[b, h])
                r = ref[idx][b, h]
                floor = 2.0 ** -20 * (np.max(np.abs(r)) + 1e-30)
                tol = 2 * (bounds[idx] + u * np.abs(r)) + floor
                err = np.abs(g - r)
                assert np.all(np.isfinite(g)), f"{name} not finite at ({b},{h})"
                ratio = float(np.max(err / tol))
                worst[name] = max(worst[name], ratio)
                assert ratio <= 1.0, f"{name} ({b},{h}): err/tol {ratio:.3f}, max err {err.max():.3e}"
                if end_to_end:
                    e = exact[idx][b, h]
                    tol_e = 2 * (bounds_e2e[idx] + u * np.abs(e)) + 2.0 ** -20 * (np.max(np.abs(e)) + 1e-30)
                    ratio_e = float(np.max(np.abs(g - e) / tol_e))
                    assert ratio_e <= 1.0, f"{name} end to end ({b},{h}): err/tol {ratio_e:.3f}"
    return worst


CASES = [
    (1, 2, 128, 128, 64, "fp16", False),
    (1, 2, 128, 128, 64, "bf16", True),
    (2, 3, 257, 257, 64, "fp16", True),
    (2, 3, 257, 257, 128, "bf16", False),
    (1, 2, 200, 300, 64, "bf16", True),     # Nq < Nk, ragged tiles
    (1, 2, 300, 130, 128, "fp16", True),    # Nq > Nk: key tile 1 sees only later queries
    (1, 1, 1, 1, 64, "fp16", False),
    (1, 2, 7, 1000, 64, "fp16", False),     # one query tile, eight key tiles
    (1, 2, 1000, 7, 128, "bf16", False),    # eight query tiles, one key tile
    (2, 2, 640, 640, 64, "fp16", True),
    (1, 2, 1000, 1000, 128, "bf16", True),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal", CASES)
def test_backward_matches_oracle(B, H, Nq, Nk, d, dtype, causal):
    q, k, v = make_qkv(B, H, Nq, Nk, d, dtype, seed=Nq * 3 + Nk + d)
    do = make_grad_out(B, H, Nq, d, dtype, seed=Nq + Nk + d)
    _check(q, k, v, do, causal, 1.0 / math.sqrt(d), dtype)


@pytest.mark.parametrize("idx", [0, 1])
def test_backward_workloads(idx):
    """The 20x20 and 40x40 YOLO workloads, every element of every gradient."""
    w = WORKLOADS[idx]
    q, k, v = make_workload_qkv(w)
    do = make_grad_out(w.B, w.H, w.Nq, w.d, w.dtype, w.seed)
    worst = _check(q, k, v, do, w.causal, w.scale, w.dtype, end_to_end=(idx == 0))
    print(f"\nBWD PARITY {w.name}: max err/tol " + ", ".join(f"{n} {r:.3f}" for n, r in worst.items()))


def test_backward_closed_forms():
    """Constant V gives dQ = dK = 0; the dV columns sum to the dO columns."""
    B, H, N, d = 1, 2, 300, 64
    q, k, _ = make_qkv(B, H, N, N, d, "bf16", seed=71)
    r = torch.randn(d, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    v = r.expand(B, H, N, d).contiguous()
    do = make_grad_out(B, H, N, d, "bf16", seed=72)
    o, lse, dq, dk, dv = _gpu_forward_backward(q, k, v, do, True, 0.125)
    # dS = P (dP - D) with dP_ij = dO_i . r = D_i exactly up to the rounding of O
    assert float(dq.abs().max()) < 5e-2 and float(dk.abs().max()) < 5e-2
    col = dv.double().sum(dim=2)  # sum over keys of dV = sum over queries of dO (P rows sum to 1)
    assert torch.allclose(col, do.double().sum(dim=2), rtol=2e-2, atol=2e-1)


def test_backward_repeatable_dk_dv():
    """dK and dV come from one CTA each and are bit-identical between calls."""
    q, k, v = (t.cuda() for t in make_qkv(2, 2, 500, 500, 64, "fp16", seed=73))
    do = make_grad_out(2, 2, 500, 64, "fp16", seed=74).cuda()
    o, lse = A.forward(q, k, v, causal=True)
    _, dk1, dv1 = A.backward(q, k, v, o, lse, do, causal=True)
    _, dk2, dv2 = A.backward(q, k, v, o, lse, do, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)


def _sampled_head(q, k, v, do, o, lse, scale, causal, u, keys, queries):
    """dK, dV of the sampled keys and dQ of the sampled queries of one (batch, head), from the
    oracle's steps on the kernel's saved o and lse, with the per-element bounds of _bounds.

    A key's dK and dV need its column of P over every query and a query's dQ its row over every
    key, so each sample is a slice of the definition computed whole."""
    nq = q.shape[0]
    qi = np.arange(nq)
    D = row_dot(do, o)
    # columns: every query against the sampled keys
    s_c = scores(q, k[keys], scale)
    if causal:
        s_c = np.where(keys[None, :] > qi[:, None], -np.inf, s_c)
    p_c = recompute_probs(s_c, lse)
    dp_c = grad_p(do, v[keys])
    ds_c = grad_scores(p_c, dp_c, D)
    dv = p_c.T @ do
    dk = scale * (ds_c.T @ q)
    e32_c = 2.0 ** -22 * np.abs(p_c) * (np.abs(do) @ np.abs(v[keys]).T + row_dot(np.abs(do), np.abs(o))[:, None])
    b_dv = 2 * u * (np.abs(p_c).T @ np.abs(do))
    b_dk = scale * (2 * u * (np.abs(ds_c).T @ np.abs(q)) + e32_c.T @ np.abs(q))
    # rows: the sampled queries against every key
    s_r = scores(q[queries], k, scale)
    if causal:
        s_r = apply_causal_mask(s_r, queries)
    p_r = recompute_probs(s_r, lse[queries])
    ds_r = grad_scores(p_r, grad_p(do[queries], v), D[queries])
    dq = scale * (ds_r @ k)
    e32_r = 2.0 ** -22 * np.abs(p_r) * (np.abs(do[queries]) @ np.abs(v).T + row_dot(np.abs(do[queries]), np.abs(o[queries]))[:, None])
    b_dq = scale * (2 * u * (np.abs(ds_r) @ np.abs(k)) + e32_r @ np.abs(k))
    return (dq, b_dq), (dk, b_dk), (dv, b_dv)


@pytest.mark.parametrize("idx", [2, 3, 4])
def test_backward_workloads_full_size_sampled(idx):
    """The 80x80, causal 2048 and 32k workloads at full size, in the launch bench.py times:
    dK and dV of 48 keys (the first and last 16 and 16 seeded ones) and dQ of 48 queries chosen
    the same way, in four (batch, head) slices, against the oracle's steps with the derived
    per-element bounds (the floor taken over the sampled elements)."""
    w = WORKLOADS[idx]
    q, k, v = make_workload_qkv(w)
    do = make_grad_out(w.B, w.H, w.Nq, w.d, w.dtype, w.seed)
    o, lse, dq, dk, dv = _gpu_forward_backward(q, k, v, do, w.causal, w.scale)
    u = UNIT[w.dtype]
    rng = np.random.default_rng(idx)
    bh = w.B * w.H
    heads = sorted({0, bh - 1} | set(int(x) for x in rng.integers(0, bh, 2)))
    worst = {"dq": 0.0, "dk": 0.0, "dv": 0.0}

    def pick(n):
        return np.unique(np.concatenate([np.arange(16), np.arange(n - 16, n), rng.integers(16, n - 16, 16)]))
    for flat in heads:
        b, h = divmod(flat, w.H)
        keys, queries = pick(w.Nk), pick(w.Nq)
        res = _sampled_head(_f64(q[b, h]), _f64(k[b, h]), _f64(v[b, h]), _f64(do[b, h]),
                            _f64(o[b, h]), _f64(lse[b, h]), w.scale, w.causal, u, keys, queries)
        got = {"dq": _f64(dq[b, h])[queries], "dk": _f64(dk[b, h])[keys], "dv": _f64(dv[b, h])[keys]}
        for name, (r, bnd) in zip(("dq", "dk", "dv"), res):
            g = got[name]
            assert np.all(np.isfinite(g)), f"{name} not finite at ({b},{h})"
            tol = 2 * (bnd + u * np.abs(r)) + 2.0 ** -20 * (np.max(np.abs(r)) + 1e-30)
            ratio = float(np.max(np.abs(g - r) / tol))
            worst[name] = max(worst[name], ratio)
            assert ratio <= 1.0, f"{name} ({b},{h}): err/tol {ratio:.3f}"
    print(f"\nBWD SAMPLED {w.name}: max err/tol " + ", ".join(f"{n} {r:.3f}" for n, r in worst.items()))
