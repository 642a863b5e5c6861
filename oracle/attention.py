"""Float64 CPU oracle for the exact scaled-dot-product attention forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this module.  The
CUDA product path never calls it and shares no code with it.

What it computes (the plain definition, no tiling):

* Attention(Q, K, V) = softmax(Q K^T / sqrt(d)) V -- "FlashAttention 深度解读"
  (coreui.cn), section "背景"; the same five-step flow in "一个反直觉的事实"
  (ai2ai.xin), section "Self-Attention的计算瓶颈": scores S = Q K^T, softmax
  of S, then softmax(S) V.
* The tiled method "does not change the mathematical definition" and is
  "not an approximation" -- YOLO11 x FlashAttention-2 (kwkr.cn), sections
  1.2 and 1.3.  So the oracle is the definition itself, in float64.
* The saved softmax statistics (section 2.3 of the same page; "log 域" in
  section "原理" of the coreui.cn page) are read as the natural-log
  logsumexp of the scaled scores: lse_i = m_i + ln(sum_j exp(s_ij - m_i)).
* The causal flag ("怎么用" on the coreui.cn page) is read as top-left
  aligned: query i may attend to key j iff j <= i.

Readings where the pages are silent are listed in the repository's design
notes; every function here is pinned by ``tests/test_oracle.py``.

Inputs may be numpy arrays or torch tensors of any float dtype; they are
upcast exactly to float64 before any arithmetic.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "to_f64", "scores", "apply_causal_mask", "softmax_rows", "weighted_sum",
    "logsumexp_rows", "attention_head_rows", "attention_f64", "attention_probs_f64",
    "brute_force", "online_softmax_f64",
]


def to_f64(x) -> np.ndarray:
    """Exact upcast of a numpy array or torch tensor to float64 numpy."""
    if hasattr(x, "detach"):  # torch tensor, possibly fp16/bf16
        import torch
        return x.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------------------
# The steps of the definition, one function each, in the pages' order.
# ---------------------------------------------------------------------------

def scores(q_rows: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Step 2 of the five-step flow: S = scale * Q K^T for a block of rows.

    q_rows: [R, d], k: [Nk, d] -> [R, Nk].
    """
    return scale * (q_rows @ k.T)


def apply_causal_mask(s: np.ndarray, row_index: np.ndarray) -> np.ndarray:
    """Set s[r, j] = -inf where key j lies after query row_index[r] (j > i)."""
    nk = s.shape[1]
    keys = np.arange(nk)[None, :]
    out = s.copy()
    out[keys > row_index[:, None]] = -np.inf
    return out


def softmax_rows(s: np.ndarray):
    """Step 3: row softmax.  Returns (P, m, l) with P = exp(s - m) / l.

    m is the row maximum and l = sum_j exp(s_j - m); subtracting the
    maximum is the fp16 safety step of "实现 3. 精度处理" on the coreui.cn
    page and leaves P unchanged mathematically.
    """
    m = np.max(s, axis=1)
    e = np.exp(s - m[:, None])
    l = np.sum(e, axis=1)
    return e / l[:, None], m, l


def weighted_sum(p: np.ndarray, v: np.ndarray) -> np.ndarray:
    """Step 4: O = P V."""
    return p @ v


def logsumexp_rows(m: np.ndarray, l: np.ndarray) -> np.ndarray:
    """Saved statistic: lse = m + ln(l), natural log of the scaled scores."""
    return m + np.log(l)


def attention_head_rows(q_rows, k, v, scale: float, causal: bool, row_index):
    """Attention for some query rows of one (batch, head).

    q_rows: [R, d]; k: [Nk, d]; v: [Nk, dv]; row_index: [R] absolute query
    indices (used only by the causal mask).  Returns (O [R, dv], lse [R]).
    Materialises the [R, Nk] block of S, as the standard method does.
    """
    q_rows = to_f64(q_rows)
    k = to_f64(k)
    v = to_f64(v)
    row_index = np.asarray(row_index, dtype=np.int64)
    s = scores(q_rows, k, scale)
    if causal:
        s = apply_causal_mask(s, row_index)
    p, m, l = softmax_rows(s)
    return weighted_sum(p, v), logsumexp_rows(m, l)


def attention_f64(q, k, v, scale: float | None = None, causal: bool = False,
                  row_block: int = 256):
    """Full attention forward in float64.

    q: [B, H, Nq, d]; k: [B, H, Nk, d]; v: [B, H, Nk, dv].
    Returns (O [B, H, Nq, dv] float64, lse [B, H, Nq] float64).
    S is materialised ``row_block`` query rows at a time so that long
    sequences fit in host memory; each block is the plain definition.
    """
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    B, H, Nq, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    o = np.empty((B, H, Nq, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, H, Nq), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for r0 in range(0, Nq, row_block):
                rows = np.arange(r0, min(Nq, r0 + row_block))
                o[b, h, rows], lse[b, h, rows] = attention_head_rows(
                    q[b, h, rows], k[b, h], v[b, h], scale, causal, rows)
    return o, lse


def attention_probs_f64(q, k, scale: float, causal: bool = False):
    """The softmax matrix P [B, H, Nq, Nk] (small inputs only)."""
    q = to_f64(q)
    k = to_f64(k)
    B, H, Nq, _ = q.shape
    out = np.empty((B, H, Nq, k.shape[2]), dtype=np.float64)
    rows = np.arange(Nq)
    for b in range(B):
        for h in range(H):
            s = scores(q[b, h], k[b, h], scale)
            if causal:
                s = apply_causal_mask(s, rows)
            out[b, h] = softmax_rows(s)[0]
    return out


# ---------------------------------------------------------------------------
# Independent second routes, used only to pin the definition above.
# ---------------------------------------------------------------------------

def brute_force(q, k, v, scale: float, causal: bool = False):
    """Pure-Python loops with math.fsum; tiny shapes only.

    Shares no arithmetic with ``attention_f64``: each output element is
    sum_j exp(s_ij - m_i) v_jc / sum_j exp(s_ij - m_i) written out.
    Returns nested lists O[b][h][i][c] and lse[b][h][i].
    """
    q = to_f64(q).tolist()
    k = to_f64(k).tolist()
    v = to_f64(v).tolist()
    out_o, out_lse = [], []
    for qb, kb, vb in zip(q, k, v):
        ob, lb = [], []
        for qh, kh, vh in zip(qb, kb, vb):
            oh, lh = [], []
            for i, qi in enumerate(qh):
                allowed = [j for j in range(len(kh)) if (not causal) or j <= i]
                s = {j: scale * math.fsum(a * b for a, b in zip(qi, kh[j])) for j in allowed}
                m = max(s.values())
                w = {j: math.exp(s[j] - m) for j in allowed}
                den = math.fsum(w.values())
                dv = len(vh[0])
                oh.append([math.fsum(w[j] * vh[j][c] for j in allowed) / den for c in range(dv)])
                lh.append(m + math.log(den))
            ob.append(oh)
            lb.append(lh)
        out_o.append(ob)
        out_lse.append(lb)
    return out_o, out_lse


def online_softmax_f64(q, k, v, scale: float, causal: bool = False, block: int = 2):
    """The pages' tiled online softmax, in float64, one K/V block at a time.

    Follows section 1.2 of the YOLO11 x FlashAttention-2 page and section
    "原理 2" / "实现 1" of the coreui.cn page: for each new K/V block,
    compute the block scores, raise the running maximum, rescale the
    already-accumulated output and exponent sum by exp(m_old - m_new), then
    add the block's exp(s - m_new) weights and their V rows.  After the last
    block divide by the sum.  Used to check that the blocked order reaches
    the same result as the definition.
    """
    q = to_f64(q)
    k = to_f64(k)
    v = to_f64(v)
    B, H, Nq, _ = q.shape
    Nk = k.shape[2]
    dv = v.shape[3]
    o = np.empty((B, H, Nq, dv))
    lse = np.empty((B, H, Nq))
    rows = np.arange(Nq)
    for b in range(B):
        for h in range(H):
            m = np.full(Nq, -np.inf)
            l = np.zeros(Nq)
            acc = np.zeros((Nq, dv))
            for j0 in range(0, Nk, block):
                kb = k[b, h, j0:j0 + block]
                vb = v[b, h, j0:j0 + block]
                s = scale * (q[b, h] @ kb.T)
                if causal:
                    keys = np.arange(j0, j0 + kb.shape[0])[None, :]
                    s = np.where(keys > rows[:, None], -np.inf, s)
                m_new = np.maximum(m, np.max(s, axis=1))
                # rows whose keys are all masked so far keep m = -inf
                safe = np.where(np.isfinite(m_new), m_new, 0.0)
                alpha = np.where(np.isfinite(m), np.exp(m - safe), 0.0)
                e = np.exp(s - safe[:, None])
                acc = acc * alpha[:, None] + e @ vb
                l = l * alpha + e.sum(axis=1)
                m = m_new
            o[b, h] = acc / l[:, None]
            lse[b, h] = m + np.log(l)
    return o, lse
