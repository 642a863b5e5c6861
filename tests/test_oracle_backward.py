"""Pins of the float64 backward oracle (CPU).

The gradients are checked against routes that share no code with
``oracle.backward``:

* central finite differences of L = sum(dO * O), with O from the forward
  oracle (itself pinned by ``tests/test_oracle.py``);
* torch float64 autograd of the attention written with torch operations;
* closed forms and invariants of the derivative: the key-gradient sums to
  zero over keys, the value-gradient sums to the summed output gradient,
  constant V has no query or key gradient, a common shift of all keys leaves
  dQ unchanged, Q = 0 gives uniform P, causal row 0 sees only key 0.

The mutation tests plant plausible mistakes in the backward steps and require
the finite-difference or closed-form pins to notice each one.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import oracle.backward as BW
from seeded_inputs import make_grad_out, make_qkv


def _rand(B, H, Nq, Nk, d, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, H, Nq, d))
    k = rng.standard_normal((B, H, Nk, d))
    v = rng.standard_normal((B, H, Nk, d))
    do = rng.standard_normal((B, H, Nq, d))
    return q, k, v, do


def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attention_f64(q, k, v, scale, causal)
    return float(np.sum(o * do))


def _finite_difference(q, k, v, do, scale, causal, eps=1e-5):
    grads = []
    for which in range(3):
        arrs = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(arrs[which])
        it = np.nditer(arrs[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in arrs]
            minus = [a.copy() for a in arrs]
            plus[which][idx] += eps
            minus[which][idx] -= eps
            g[idx] = (_loss(*plus, do, scale, causal) - _loss(*minus, do, scale, causal)) / (2 * eps)
        grads.append(g)
    return grads


def _torch_grads(q, k, v, do, scale, causal):
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    s = scale * qt @ kt.transpose(-1, -2)
    if causal:
        nq, nk = s.shape[-2:]
        hide = torch.arange(nk)[None, :] > torch.arange(nq)[:, None]
        s = s.masked_fill(hide, float("-inf"))
    o = torch.softmax(s, dim=-1) @ vt
    (o * torch.tensor(do)).sum().backward()
    return qt.grad.numpy(), kt.grad.numpy(), vt.grad.numpy()


def _max_err(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))))


# ------------------------------------------------------------------ pins

def fd_pin(causal):
    q, k, v, do = _rand(1, 1, 4, 5, 3, seed=11 + causal)
    scale = 0.7
    got = oracle.attention_backward_f64(q, k, v, do, scale, causal)
    want = _finite_difference(q, k, v, do, scale, causal)
    return max(_max_err(g, w) for g, w in zip(got, want))


def invariant_failures():
    """Names of the closed-form pins the current backward violates."""
    bad = []
    q, k, v, do = _rand(2, 2, 6, 6, 4, seed=5)
    for causal in (False, True):
        dq, dk, dv = oracle.attention_backward_f64(q, k, v, do, 0.5, causal)
        if _max_err(dk.sum(axis=2), 0.0) > 1e-12:
            bad.append(f"sum_j dK = 0 (causal={causal})")
        if _max_err(dv.sum(axis=2), do.sum(axis=2)) > 1e-12:
            bad.append(f"sum_j dV = sum_i dO (causal={causal})")
        vc = np.broadcast_to(v[:, :, :1, :], v.shape).copy()
        dq0, dk0, _ = oracle.attention_backward_f64(q, k, vc, do, 0.5, causal)
        if max(_max_err(dq0, 0.0), _max_err(dk0, 0.0)) > 1e-12:
            bad.append(f"constant V: dQ = dK = 0 (causal={causal})")
        u = np.random.default_rng(3).standard_normal(4)
        dq_shift, _, _ = oracle.attention_backward_f64(q, k + u, v, do, 0.5, causal)
        if _max_err(dq_shift, dq) > 1e-11:
            bad.append(f"dQ invariant under a common key shift (causal={causal})")
        if causal and _max_err(dq[:, :, 0], 0.0) > 1e-12:
            bad.append("causal row 0: dQ_0 = 0")
    # Q = 0, non-causal: P is uniform, so every key's dV is the mean of dO over queries
    qz = np.zeros_like(q)
    _, _, dvz = oracle.attention_backward_f64(qz, k, v, do, 0.5, False)
    want = np.broadcast_to(do.sum(axis=2, keepdims=True) / k.shape[2], dvz.shape)
    if _max_err(dvz, want) > 1e-12:
        bad.append("Q = 0: dV_j = sum_i dO_i / Nk")
    return bad


# ------------------------------------------------------------------ tests

@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(causal):
    assert fd_pin(causal) < 1e-7


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [(1, 2, 7, 9, 5), (2, 1, 16, 16, 8)])
def test_torch_autograd(causal, shape):
    q, k, v, do = _rand(*shape, seed=sum(shape) + causal)
    scale = 1.0 / math.sqrt(shape[-1])
    got = oracle.attention_backward_f64(q, k, v, do, scale, causal)
    want = _torch_grads(q, k, v, do, scale, causal)
    for g, w in zip(got, want):
        assert _max_err(g, w) < 1e-10


def test_closed_forms_and_invariants():
    assert invariant_failures() == []


def test_saved_statistics_path_matches_fresh_forward():
    q, k, v = make_qkv(1, 2, 150, 200, 64, "bf16", seed=9)
    do = make_grad_out(1, 2, 150, 64, "bf16", seed=9)
    o, lse = oracle.attention_f64(q, k, v, 0.125, True)
    a = oracle.attention_backward_f64(q, k, v, do, 0.125, True, o=o, lse=lse)
    b = oracle.attention_backward_f64(q, k, v, do, 0.125, True)
    for x, y in zip(a, b):
        assert _max_err(x, y) == 0.0


def test_seeded_grad_out_is_deterministic():
    a = make_grad_out(2, 3, 17, 64, "fp16", seed=4)
    b = make_grad_out(2, 3, 17, 64, "fp16", seed=4)
    assert a.dtype == torch.float16 and a.shape == (2, 3, 17, 64) and torch.equal(a, b)


# ------------------------------------------------------------------ mutations

def _ds_without_rowdot(p, dp, dsum):
    return p * dp


def _ds_wrong_sign(p, dp, dsum):
    return p * (dsum[:, None] - dp)


def _dq_no_scale(ds, k, scale):
    return ds @ k


def _dk_transposed(ds, q, scale):
    return scale * (ds @ q)


def _dv_transposed(p, do):
    return p @ do


def _rowdot_without_o(do, o):
    return np.sum(do, axis=1)


def _probs_base2(s, lse):
    return np.exp2(s - lse[:, None])


def _no_mask(s, row_index):
    return s


MUTATIONS = [
    ("grad_scores", _ds_without_rowdot),
    ("grad_scores", _ds_wrong_sign),
    ("grad_q", _dq_no_scale),
    ("grad_k", _dk_transposed),
    ("grad_v", _dv_transposed),
    ("row_dot", _rowdot_without_o),
    ("recompute_probs", _probs_base2),
    ("apply_causal_mask", _no_mask),
]


@pytest.mark.parametrize("name,fn", MUTATIONS, ids=[f.__name__ for _, f in MUTATIONS])
def test_pins_catch_planted_mistakes(monkeypatch, name, fn):
    monkeypatch.setattr(BW, name, fn)
    caught = bool(invariant_failures())
    if not caught:
        caught = fd_pin(False) > 1e-6 or fd_pin(True) > 1e-6
    assert caught, f"no pin noticed the mutation of {name}"
