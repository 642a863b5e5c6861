"""GPU parity of the FP8 (e4m3) forward against the float64 oracle on the dequantised inputs.

The kernel rounds P to e4m3 before the P V product, so unlike the 16-bit
forward its error grows with the data.  The bar is derived per element from
that arithmetic (P and V are oracle quantities of the dequantised inputs):

* P rounding: an e4m3 value x (|x| < 448) is within 2^-4 |x| + 2^-10 of the
  fp32 value it rounds (3 mantissa bits; subnormal spacing 2^-9).  P enters
  the P V product relative to the running row max (the kernel's frame, where
  every P lies in [0, 256) and the row sum l' >= 1), so the O error is at most
  2^-4 (P|V|)_ic + 2^-10 sum_j |V_jc| / l' <= 2^-4 A + 2^-10 B with
  A = sum_j P_ij |V_jc| and B = max_j P_ij sum_j |V_jc| (1 / l = max_j P_ij).
* exponentials: ex2.approx and the FMA-pipe polynomial (relative 7.5e-5) add
  1e-4 A; fp32 accumulation of the products adds 2^-11 A; the score sums may
  err by 2^-12 scale (|Q||K|^T)_ij = dx_ij, moving P by a factor exp(dx):
  dx_max (A + |O|).
* bf16 rounding of O: 2^-8 |O|.
Bar: 2 (2^-4 A + 2^-10 B + (2^-11 + 1e-4) A + dx_max (A + |O|)) + 2^-7 |O| + 1e-6.
lse: 1e-3 + 2 dx_max.

An elementwise worst case is loose when many keys share the weight, so each
case also checks the root-mean-square error against the rounding-noise model:
independent roundings of variance 2^-8 / 3 (relative) or 2^-20 / 3
(absolute) give E[err^2] <= sum_j (2^-8/3 P_ij^2 + 2^-20/3 (max_j P_ij)^2) V_jc^2
+ 2^-16/3 O^2; the measured mean square must stay below 4 times the model's
(a wrong key order inside a packed word, a swapped operand or a dropped
descale overshoots it by one to several orders of magnitude).
"""
import math

import numpy as np
import pytest
import torch

import exact_attention_153_b200 as A
import oracle
from exact_attention_153_b200 import build_lib
from seeded_inputs import make_fp8_qkv

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    build_lib.build()
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _head_reference(q8, k8, vt8, descales, b, h, scale, causal, rows):
    """Oracle O, lse and the bound terms for some query rows of one (batch, head)."""
    qs, ks, vs = descales
    q = oracle.dequantize_e4m3(q8[b, h, rows], qs)
    k = oracle.dequantize_e4m3(k8[b, h], ks)
    v = oracle.untranspose_v(oracle.dequantize_e4m3(vt8[b, h], vs))
    s = oracle.scores(q, k, scale)
    if causal:
        s = oracle.apply_causal_mask(s, rows)
    p, m, l = oracle.softmax_rows(s)
    o = oracle.weighted_sum(p, v)
    lse = oracle.logsumexp_rows(m, l)
    absv = np.abs(v)
    a = p @ absv
    pmax = p.max(axis=1, keepdims=True)
    bterm = pmax * absv.sum(axis=0, keepdims=True)
    dx = 2.0 ** -12 * scale * (np.abs(q) @ np.abs(k).T)
    if causal:
        dx = np.where(np.isfinite(s), dx, 0.0)
    dx_max = dx.max(axis=1, keepdims=True)
    var = (2.0 ** -8 / 3) * ((p * p) @ (v * v)) + (2.0 ** -20 / 3) * pmax ** 2 * (v * v).sum(0) \
        + (2.0 ** -16 / 3) * o * o
    tol = 2 * (2.0 ** -4 * a + 2.0 ** -10 * bterm + (2.0 ** -11 + 1e-4) * a
               + dx_max * (a + np.abs(o))) + 2.0 ** -7 * np.abs(o) + 1e-6
    return o, lse, tol, 1e-3 + 2 * dx_max[:, 0], var


def _check(o_gpu, lse_gpu, q8, k8, vt8, descales, scale, causal, heads, rows_of):
    """Every listed (b, h) at rows_of(b, h): elementwise bar and the noise-model RMS check."""
    se, sv, worst = 0.0, 0.0, 0.0
    for b, h in heads:
        rows = rows_of(b, h)
        o, lse, tol, ltol, var = _head_reference(q8, k8, vt8, descales, b, h, scale, causal, rows)
        og = o_gpu[b, h, rows].double().numpy()
        lg = lse_gpu[b, h, rows].double().numpy()
        err = np.abs(og - o)
        assert np.isfinite(og).all() and np.isfinite(lg).all()
        bad = err > tol
        assert not bad.any(), (f"(b,h)=({b},{h}): {int(bad.sum())} elements over the bar, "
                               f"max err {err.max():.3e}, max ratio {(err / tol).max():.2f}")
        lerr = np.abs(lg - lse)
        assert (lerr <= ltol).all(), f"lse err {lerr.max():.3e}"
        se += float((err * err).sum())
        sv += float(var.sum())
        worst = max(worst, float((err / tol).max()))
    assert se <= 4 * sv, f"mean square error {se:.3e} vs noise model {sv:.3e}"
    return worst, math.sqrt(se / sv)


def _run(B, H, Nq, Nk, causal, seed, qk_scale=1.0, split=None):
    q8, k8, vt8, ds = make_fp8_qkv(B, H, Nq, Nk, 128, seed, qk_scale)
    qd, kd, vd = q8.cuda(), k8.cuda(), vt8.cuda()
    ws = A.workspace_for(qd, kd, causal)
    if split is not None:
        assert (ws is not None) == split
    o, lse = A.forward_fp8(qd, kd, vd, ds, causal=causal, workspace=ws)
    torch.cuda.synchronize()
    st, word = A.attn_get_device_status()
    assert st == 0, f"device status {word:#x}"
    return q8, k8, vt8, ds, o.cpu(), lse.cpu()


SHAPES = [
    (1, 1, 128, 128, False),    # one tile
    (1, 1, 1, 16, False),       # one query, the smallest key count
    (2, 3, 300, 512, False),    # ragged query tiles, several key tiles
    (1, 2, 1000, 1008, True),   # causal, ragged on both axes, Nq != Nk
    (1, 1, 77, 2000, True),     # causal with far more keys than queries
    (16, 4, 1600, 1600, False), # 40x40 YOLO shape at d = 128: dual units
    (3, 2, 640, 2048, False),
]


@pytest.mark.parametrize("B,H,Nq,Nk,causal", SHAPES)
def test_fp8_parity(B, H, Nq, Nk, causal):
    q8, k8, vt8, ds, o, lse = _run(B, H, Nq, Nk, causal, seed=B * 1000 + Nq + Nk)
    heads = [(b, h) for b in range(B) for h in range(H)]
    _check(o, lse, q8, k8, vt8, ds, 1 / math.sqrt(128), causal, heads, lambda b, h: np.arange(Nq))


@pytest.mark.parametrize("B,H,N,causal", [(1, 1, 4096, False), (1, 2, 4096, True),
                                          (1, 1, 3504, False)])
def test_fp8_split_mode(B, H, N, causal):
    """Few units with many key tiles: split mode, pieces merged in the log domain."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert A.attn_plan(B, H, N, N, 128, int(causal), sms)["split"] == 1
    q8, k8, vt8, ds, o, lse = _run(B, H, N, N, causal, seed=N + 3, split=True)
    heads = [(b, h) for b in range(B) for h in range(H)]
    _check(o, lse, q8, k8, vt8, ds, 1 / math.sqrt(128), causal, heads, lambda b, h: np.arange(N))


def test_fp8_long_context_sampled():
    """The long-context shape (1 x 32 heads x 32768, causal, Q and K x 0.5) at full size:
    per head the first, 64 random and the last 64 query rows, all 32768 keys each."""
    B, H, N = 1, 32, 32768
    q8, k8, vt8, ds, o, lse = _run(B, H, N, N, True, seed=1005, qk_scale=0.5)
    rng = np.random.default_rng(7)

    def rows_of(b, h):
        return np.unique(np.concatenate([np.arange(64), rng.integers(64, N - 64, 64),
                                         np.arange(N - 64, N)]))
    worst, rms_ratio = _check(o, lse, q8, k8, vt8, ds, 1 / math.sqrt(128), True,
                              [(0, h) for h in range(H)], rows_of)
    print(f"long context fp8: worst err/bar {worst:.3f}, rms/model {rms_ratio:.3f}")


def test_fp8_dominant_key():
    """One key per row far above the rest: O must be that key's V row (P rounding is exact
    at 1 and tiny elsewhere), which a mis-ordered P or V cannot reproduce."""
    B, H, N = 1, 2, 512
    q8, k8, vt8, ds = make_fp8_qkv(B, H, N, N, 128, seed=21)
    # key j = (7 i + 3) % N gets q_i itself (scaled up): its score dominates row i
    qf = q8.to(torch.float32)
    kf = k8.to(torch.float32) * 0.05
    perm = (7 * torch.arange(N) + 3) % N
    kf[:, :, perm] = qf[:, :, :N]
    k8 = kf.to(torch.float8_e4m3fn)
    ds = (ds[0], ds[1], ds[2])
    scale = 4.0 / math.sqrt(128)
    qd, kd, vd = q8.cuda(), k8.cuda(), vt8.cuda()
    o, lse = A.forward_fp8(qd, kd, vd, ds, scale=scale)
    torch.cuda.synchronize()
    o = o.cpu()
    _check(o, lse.cpu(), q8, k8, vt8, ds, scale, False, [(0, 0), (0, 1)],
           lambda b, h: np.arange(N))
    v = oracle.untranspose_v(oracle.dequantize_e4m3(vt8, ds[2]))
    picked = v[:, :, perm.numpy()]
    assert np.abs(o.double().numpy() - picked).max() < 0.05 * np.abs(picked).max()


def test_fp8_repeatable():
    """Two calls give the same bits, in split mode (pieces merged in a fixed order) and in
    unit mode."""
    B, H, N = 1, 1, 4096
    q8, k8, vt8, ds = make_fp8_qkv(B, H, N, N, 128, seed=99)
    qd, kd, vd = q8.cuda(), k8.cuda(), vt8.cuda()
    ws = A.workspace_for(qd, kd, False)
    assert ws is not None
    o1, l1 = A.forward_fp8(qd, kd, vd, ds, workspace=ws)
    o2, l2 = A.forward_fp8(qd, kd, vd, ds, workspace=ws)
    o3, l3 = A.forward_fp8(qd, kd, vd, ds)
    o4, l4 = A.forward_fp8(qd, kd, vd, ds)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o3, o4) and torch.equal(l3, l4)


def test_fp8_rejects_bad_arguments_on_device():
    q8, k8, vt8, ds = make_fp8_qkv(1, 1, 64, 64, 128, seed=1)
    qd, kd, vd = q8.cuda(), k8.cuda(), vt8.cuda()
    o = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device="cuda")
    # misaligned output: ATTN_ERR_ALIGN, nothing written
    o_big = torch.zeros(64 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    st = A.attn_fwd_fp8(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o_big.data_ptr() + 2, None,
                        1, 1, 64, 64, 128, 0.1, *ds, 0, None, 0, 0)
    assert st == 5
    st = A.attn_fwd_fp8(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), None,
                        1, 1, 64, 64, 128, 0.1, ds[0], -1.0, ds[2], 0, None, 0, 0)
    assert st == 6
    torch.cuda.synchronize()
    assert int(o.float().abs().sum()) == 0 and int(o_big.float().abs().sum()) == 0
