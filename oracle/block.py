"""Float64 CPU oracle for the attention block around the attention forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
CUDA product path never calls it and shares no code with it.

What it computes: the attention module of YOLO11 x FlashAttention-2
(kwkr.cn), section 2.2, for an input x [B, N, C] with C = H * d:

* qkv = x W_qkv^T (+ b_qkv): the qkv Linear(dim, 3 * dim) (the page builds
  it without a bias; an optional bias is accepted here);
* its [B, N, 3 C] output read as [B, N, 3, H, d]; taking index 0, 1, 2 of
  the third axis and swapping the N and H axes gives q, k, v [B, H, N, d];
* o = attention(q, k, v) (``oracle.attention.attention_f64``);
* o transposed back to [B, N, H, d], read as [B, N, C], then the proj
  Linear(dim, dim): y = o' W_o^T + b_o.

Every step is one function below, in that order; every function is pinned
by ``tests/test_oracle_block.py``.
"""
from __future__ import annotations

import numpy as np

from .attention import attention_f64, to_f64

__all__ = ["linear", "split_qkv", "merge_heads", "attention_block_f64"]


def linear(x, w, b=None) -> np.ndarray:
    """y = x W^T (+ b) over the last axis: x [..., K], W [N_out, K], b [N_out]."""
    y = to_f64(x) @ to_f64(w).T
    if b is not None:
        y = y + to_f64(b)
    return y


def split_qkv(qkv: np.ndarray, H: int, d: int):
    """[B, N, 3 H d] -> q, k, v [B, H, N, d]: the reshape to [B, N, 3, H, d],
    the unbind of axis 2 and the transpose of axes 1 and 2."""
    B, N, _ = qkv.shape
    r = qkv.reshape(B, N, 3, H, d)
    return tuple(np.ascontiguousarray(r[:, :, i].transpose(0, 2, 1, 3)) for i in range(3))


def merge_heads(o: np.ndarray) -> np.ndarray:
    """[B, H, N, d] -> [B, N, H d]: the transpose back and the reshape."""
    B, H, N, d = o.shape
    return np.ascontiguousarray(o.transpose(0, 2, 1, 3)).reshape(B, N, H * d)


def attention_block_f64(x, w_qkv, b_qkv, w_o, b_o, H: int, d: int, scale=None,
                        causal: bool = False):
    """The whole block in float64.  Returns (y, q, k, v, o, lse)."""
    qkv = linear(x, w_qkv, b_qkv)
    q, k, v = split_qkv(qkv, H, d)
    o, lse = attention_f64(q, k, v, scale, causal)
    y = linear(merge_heads(o), w_o, b_o)
    return y, q, k, v, o, lse
