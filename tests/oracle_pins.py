"""Pins of the float64 oracle against facts that do not come from the oracle.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
a closed form, an invariant, brute force or a library routine.  They call
the oracle through ``oracle.attention`` attributes at call time, so the
mutation tests can plant a mistake in one step and check that some pin
notices.

The pages print no worked input/output example (no values to copy), so the
pins are closed forms and invariants that the definition
softmax(Q K^T * scale) V fixes -- "FlashAttention 深度解读" (coreui.cn),
section "背景" -- plus brute force and torch's float64 SDPA, the entry point
the YOLO11 x FlashAttention-2 page (kwkr.cn) calls in section 2.2.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle.attention as A

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * scale


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"
    return err


# --- hand-worked cases from tests/golden ------------------------------------

def pin_hand_examples():
    """Closed-form two-key cases whose weights are 1/3 and 2/3 (see fixture)."""
    with open(os.path.join(GOLDEN, "hand_examples.json"), encoding="utf-8") as f:
        cases = json.load(f)["cases"]
    for c in cases:
        q = np.array(c["q"], dtype=np.float64)[None, None]
        k = np.array(c["k"], dtype=np.float64)[None, None]
        v = np.array(c["v"], dtype=np.float64)[None, None]
        o, lse = A.attention_f64(q, k, v, c["scale"], c["causal"])
        o_exp = np.array(c["o"], dtype=np.float64)
        lse_exp = np.array([eval(x, {"ln": math.log}) for x in c["lse"]])
        _close(o[0, 0], o_exp, 1e-13, c["name"] + " O")
        _close(lse[0, 0], lse_exp, 1e-13, c["name"] + " lse")


# --- invariants and closed forms --------------------------------------------

def pin_row_sums():
    """Every softmax row sums to one."""
    for causal in (False, True):
        q = _rand((2, 2, 9, 8), 1)
        k = _rand((2, 2, 9, 8), 2)
        p = A.attention_probs_f64(q, k, 0.35, causal)
        _close(p.sum(-1), np.ones(p.shape[:-1]), 1e-12, f"row sums causal={causal}")
        assert np.all(p >= 0.0), "negative probability"


def pin_constant_v():
    """All V rows equal r  =>  every output row equals r."""
    for causal in (False, True):
        q = _rand((1, 2, 7, 8), 3)
        k = _rand((1, 2, 11, 8), 4)
        r = _rand((8,), 5)
        v = np.broadcast_to(r, (1, 2, 11, 8)).copy()
        o, _ = A.attention_f64(q, k, v, 0.4, causal)
        _close(o, np.broadcast_to(r, o.shape), 1e-12, f"constant V causal={causal}")


def pin_q_zero():
    """Q = 0: O_i is the mean of the visible V rows and lse_i = ln(#visible)."""
    nk = 13
    k = _rand((1, 1, nk, 4), 6)
    v = _rand((1, 1, nk, 3), 7)
    q = np.zeros((1, 1, nk, 4))
    o, lse = A.attention_f64(q, k, v, 0.5, False)
    _close(o[0, 0], np.broadcast_to(v[0, 0].mean(0), (nk, 3)), 1e-12, "Q=0 O")
    _close(lse[0, 0], np.full(nk, math.log(nk)), 1e-12, "Q=0 lse")
    o, lse = A.attention_f64(q, k, v, 0.5, True)
    prefix = np.cumsum(v[0, 0], axis=0) / np.arange(1, nk + 1)[:, None]
    _close(o[0, 0], prefix, 1e-12, "Q=0 causal O")
    _close(lse[0, 0], np.log(np.arange(1, nk + 1)), 1e-12, "Q=0 causal lse")


def pin_dominant_key():
    """A key aligned with q_i and much longer than the rest takes all of row i."""
    q = _rand((1, 1, 5, 16), 8)
    k = _rand((1, 1, 9, 16), 9)
    v = _rand((1, 1, 9, 16), 10)
    scale = 0.25
    for i, jstar in [(0, 3), (2, 7), (4, 0)]:
        kk = k.copy()
        qi = q[0, 0, i]
        kk[0, 0, jstar] = 400.0 * qi / np.linalg.norm(qi)  # gap >= 60 in the exponent
        o, _ = A.attention_f64(q, kk, v, scale, False)
        _close(o[0, 0, i], v[0, 0, jstar], 1e-12, f"dominant key row {i}")


def pin_causal_row0():
    """Causal row 0 sees only key 0: O_0 = V_0 and lse_0 = scale q_0 . k_0."""
    q = _rand((2, 3, 6, 8), 11)
    k = _rand((2, 3, 6, 8), 12)
    v = _rand((2, 3, 6, 8), 13)
    o, lse = A.attention_f64(q, k, v, 0.3, True)
    _close(o[:, :, 0], v[:, :, 0], 1e-12, "causal row 0 O")
    _close(lse[:, :, 0], 0.3 * np.einsum("bhd,bhd->bh", q[:, :, 0], k[:, :, 0]),
           1e-12, "causal row 0 lse")


def pin_single_key():
    """Nk = 1: every row returns V_0; lse_i = scale q_i . k_0."""
    q = _rand((1, 2, 5, 8), 14)
    k = _rand((1, 2, 1, 8), 15)
    v = _rand((1, 2, 1, 8), 16)
    o, lse = A.attention_f64(q, k, v, 0.7, False)
    _close(o, np.broadcast_to(v, o.shape), 1e-12, "Nk=1 O")
    _close(lse, 0.7 * np.einsum("bhid,bhd->bhi", q, k[:, :, 0]), 1e-12, "Nk=1 lse")


def pin_permutation():
    """Non-causal: permuting K and V rows together leaves O and lse unchanged."""
    q = _rand((1, 2, 6, 8), 17)
    k = _rand((1, 2, 10, 8), 18)
    v = _rand((1, 2, 10, 8), 19)
    perm = np.random.default_rng(20).permutation(10)
    o1, l1 = A.attention_f64(q, k, v, 0.3, False)
    o2, l2 = A.attention_f64(q, k[:, :, perm], v[:, :, perm], 0.3, False)
    _close(o1, o2, 1e-12, "permutation O")
    _close(l1, l2, 1e-12, "permutation lse")


def pin_key_shift():
    """Adding u to every key keeps O and shifts lse_i by scale q_i . u."""
    for causal in (False, True):
        q = _rand((1, 2, 7, 8), 21)
        k = _rand((1, 2, 7, 8), 22)
        v = _rand((1, 2, 7, 8), 23)
        u = _rand((8,), 24)
        o1, l1 = A.attention_f64(q, k, v, 0.3, causal)
        o2, l2 = A.attention_f64(q, k + u, v, 0.3, causal)
        _close(o1, o2, 1e-12, f"key shift O causal={causal}")
        _close(l2 - l1, 0.3 * (q @ u), 1e-12, f"key shift lse causal={causal}")


def pin_online_blocked():
    """The pages' blocked online softmax reaches the one-shot definition."""
    for causal in (False, True):
        for block in (1, 2, 3, 5):
            q = _rand((1, 2, 9, 8), 25, 2.0)
            k = _rand((1, 2, 9, 8), 26, 2.0)
            v = _rand((1, 2, 9, 8), 27)
            o1, l1 = A.attention_f64(q, k, v, 0.5, causal)
            o2, l2 = A.online_softmax_f64(q, k, v, 0.5, causal, block)
            _close(o1, o2, 1e-13, f"online block={block} causal={causal} O")
            _close(l1, l2, 1e-13, f"online block={block} causal={causal} lse")


# --- second routes: brute force and a library routine ------------------------

def pin_brute_force():
    """Pure-Python fsum loops agree with the numpy oracle to 1e-12."""
    shapes = [(1, 1, 1, 1, 1), (2, 2, 3, 5, 4), (1, 2, 8, 3, 8), (2, 1, 17, 17, 4),
              (1, 1, 5, 2, 8)]
    for n, (B, H, Nq, Nk, d) in enumerate(shapes):
        for causal in (False, True):
            q = _rand((B, H, Nq, d), 100 + n)
            k = _rand((B, H, Nk, d), 200 + n)
            v = _rand((B, H, Nk, d), 300 + n)
            scale = 1.0 / math.sqrt(d)
            o1, l1 = A.attention_f64(q, k, v, scale, causal)
            o2, l2 = A.brute_force(q, k, v, scale, causal)
            _close(o1, np.array(o2), 1e-12, f"brute {B, H, Nq, Nk, d} causal={causal} O")
            _close(l1, np.array(l2), 1e-12, f"brute {B, H, Nq, Nk, d} causal={causal} lse")


def pin_torch_sdpa():
    """torch's float64 CPU scaled_dot_product_attention agrees to 1e-10."""
    for n, (B, H, Nq, Nk, d) in enumerate([(2, 3, 33, 33, 16), (1, 2, 20, 45, 8),
                                           (1, 1, 64, 64, 64)]):
        for causal in (False, True):
            if causal and Nq != Nk:
                continue
            q = _rand((B, H, Nq, d), 400 + n)
            k = _rand((B, H, Nk, d), 500 + n)
            v = _rand((B, H, Nk, d), 600 + n)
            scale = 1.0 / math.sqrt(d)
            o1, _ = A.attention_f64(q, k, v, scale, causal)
            o2 = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
                is_causal=causal, scale=scale).numpy()
            _close(o1, o2, 1e-10, f"torch sdpa {B, H, Nq, Nk, d} causal={causal}")


INDEPENDENT_PINS = [
    pin_hand_examples, pin_row_sums, pin_constant_v, pin_q_zero, pin_dominant_key,
    pin_causal_row0, pin_single_key, pin_permutation, pin_key_shift, pin_online_blocked,
]
ROUTE_PINS = [pin_brute_force, pin_torch_sdpa]
ALL_PINS = INDEPENDENT_PINS + ROUTE_PINS
