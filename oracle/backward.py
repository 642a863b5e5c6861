"""Float64 CPU oracle for the gradients of the exact attention forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
CUDA product path never calls it and shares no code with it.

What the pages fix: training runs a backward pass that does not cache the
softmax matrix but recomputes it from the statistics the forward saved --
"YOLOv12推理速度翻倍秘诀：Flash Attention加持" (0539edu.com), section 1
(recompute the softmax intermediates in the backward pass instead of storing
them); YOLO11 x FlashAttention-2 (kwkr.cn), section 2.3 (training keeps the
statistics the backward needs) and section 4.3 (recomputation recomputes the
attention statistics).  The pages do not write the gradient out; it is the
derivative of the forward definition.  With L a scalar function of the
output and dO = dL/dO, for one (batch, head), in float64:

    S  = scale * Q K^T   (-inf where the causal mask hides a key)
    P  = exp(S - lse)    (the softmax, recomputed from the saved lse)
    O  = P V
    dV = P^T dO
    dP = dO V^T
    D  = rowsum(dO * O)  (= rowsum(P * dP))
    dS = P * (dP - D)    (the softmax Jacobian applied to dP, row by row)
    dQ = scale * dS K
    dK = scale * dS^T Q

Each step is one function below, in that order; ``attention_backward_f64``
chains them.  Every function is pinned by ``tests/test_oracle_backward.py``.
"""
from __future__ import annotations

import math

import numpy as np

from .attention import apply_causal_mask, attention_f64, scores, to_f64

__all__ = [
    "recompute_probs", "grad_v", "grad_p", "row_dot", "grad_scores", "grad_q", "grad_k",
    "attention_backward_f64",
]


def recompute_probs(s: np.ndarray, lse: np.ndarray) -> np.ndarray:
    """P = exp(S - lse) from the saved natural-log statistics (masked entries give 0)."""
    return np.exp(s - lse[:, None])


def grad_v(p: np.ndarray, do: np.ndarray) -> np.ndarray:
    """dV = P^T dO: [Nq, Nk] x [Nq, dv] -> [Nk, dv]."""
    return p.T @ do


def grad_p(do: np.ndarray, v: np.ndarray) -> np.ndarray:
    """dP = dO V^T: [Nq, dv] x [Nk, dv] -> [Nq, Nk]."""
    return do @ v.T


def row_dot(do: np.ndarray, o: np.ndarray) -> np.ndarray:
    """D_i = sum_c dO_ic O_ic."""
    return np.sum(do * o, axis=1)


def grad_scores(p: np.ndarray, dp: np.ndarray, dsum: np.ndarray) -> np.ndarray:
    """dS = P * (dP - D): row i of the softmax Jacobian, diag(P_i) - P_i P_i^T, times dP_i."""
    return p * (dp - dsum[:, None])


def grad_q(ds: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """dQ = scale * dS K."""
    return scale * (ds @ k)


def grad_k(ds: np.ndarray, q: np.ndarray, scale: float) -> np.ndarray:
    """dK = scale * dS^T Q."""
    return scale * (ds.T @ q)


def attention_backward_f64(q, k, v, do, scale: float | None = None, causal: bool = False,
                           o=None, lse=None):
    """Gradients (dQ, dK, dV) of the attention forward for the output gradient dO.

    q: [B, H, Nq, d]; k: [B, H, Nk, d]; v: [B, H, Nk, dv]; do: [B, H, Nq, dv].
    ``o`` and ``lse`` are the forward's output and saved statistics; when not
    given they are computed by the forward oracle.  Returns float64 arrays
    shaped like q, k and v.  Materialises the [Nq, Nk] matrices of one head
    at a time (small and medium shapes).
    """
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    do = to_f64(do)
    B, H, Nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if o is None or lse is None:
        o, lse = attention_f64(q, k, v, scale, causal)
    o = to_f64(o)
    lse = to_f64(lse)
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    rows = np.arange(Nq)
    for b in range(B):
        for h in range(H):
            s = scores(q[b, h], k[b, h], scale)
            if causal:
                s = apply_causal_mask(s, rows)
            p = recompute_probs(s, lse[b, h])
            dv[b, h] = grad_v(p, do[b, h])
            dp = grad_p(do[b, h], v[b, h])
            ds = grad_scores(p, dp, row_dot(do[b, h], o[b, h]))
            dq[b, h] = grad_q(ds, k[b, h], scale)
            dk[b, h] = grad_k(ds, q[b, h], scale)
    return dq, dk, dv
