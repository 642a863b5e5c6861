"""Pins of the block oracle (oracle/block.py) on the CPU.

* an independent route: torch float64 ops written the way the page's module
  writes them (F.linear, reshape (B, N, 3, H, d), unbind(2), transpose(1, 2),
  scaled_dot_product_attention, transpose(1, 2).reshape(B, N, C), F.linear);
* closed forms: every element of the split lands where its column index
  says, merge undoes the split, identity weights pass x through, a block
  whose V is zero outputs the proj bias, a block whose Q is zero outputs the
  key mean of V through the proj;
* planted mistakes (axis order of the split, a missing transpose, W instead of
  W^T, a dropped bias) are each caught by the closed forms alone.
"""
import numpy as np
import pytest
import torch

import oracle.block as Bk

RNG = np.random.default_rng(11)


def _case(B=2, N=5, H=3, d=4, C_out=None):
    C = H * d
    C_out = C if C_out is None else C_out
    x = RNG.standard_normal((B, N, C))
    w_qkv = RNG.standard_normal((3 * C, C)) / np.sqrt(C)
    b_qkv = RNG.standard_normal(3 * C)
    w_o = RNG.standard_normal((C_out, C)) / np.sqrt(C)
    b_o = RNG.standard_normal(C_out)
    return x, w_qkv, b_qkv, w_o, b_o


@pytest.mark.parametrize("causal", [False, True])
def test_matches_the_page_module_in_torch(causal):
    B, N, H, d = 2, 7, 3, 4
    x, w_qkv, b_qkv, w_o, b_o = _case(B, N, H, d, C_out=9)
    y, q, k, v, o, lse = Bk.attention_block_f64(x, w_qkv, b_qkv, w_o, b_o, H, d, 0.37, causal)
    tx = torch.from_numpy(x)
    qkv = torch.nn.functional.linear(tx, torch.from_numpy(w_qkv), torch.from_numpy(b_qkv))
    qkv = qkv.reshape(B, N, 3, H, d)
    tq, tk, tv = qkv.unbind(2)
    tq, tk, tv = tq.transpose(1, 2), tk.transpose(1, 2), tv.transpose(1, 2)
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=0.37)
    ty = torch.nn.functional.linear(to.transpose(1, 2).reshape(B, N, H * d),
                                    torch.from_numpy(w_o), torch.from_numpy(b_o))
    for a, b in ((q, tq), (k, tk), (v, tv), (o, to), (y, ty)):
        assert np.max(np.abs(a - b.numpy())) < 1e-10


def _pin_split(split_qkv):
    B, N, H, d = 2, 3, 2, 4
    C = H * d
    codes = np.zeros((B, N, 3 * C))
    for b in range(B):
        for n in range(N):
            for c in range(3 * C):
                codes[b, n, c] = 1000 * b + 100 * n + c
    q, k, v = split_qkv(codes, H, d)
    for which, t in enumerate((q, k, v)):
        assert t.shape == (B, H, N, d)
        for b in range(B):
            for h in range(H):
                for n in range(N):
                    for dd in range(d):
                        assert t[b, h, n, dd] == 1000 * b + 100 * n + which * C + h * d + dd


def _pin_merge(split_qkv, merge_heads):
    B, N, H, d = 2, 5, 3, 4
    qkv = RNG.standard_normal((B, N, 3 * H * d))
    q, _, v = split_qkv(qkv, H, d)
    assert np.array_equal(merge_heads(q), qkv[:, :, :H * d])
    assert np.array_equal(merge_heads(v), qkv[:, :, 2 * H * d:])


def _pin_linear(linear):
    x = RNG.standard_normal((2, 3, 5))
    assert np.allclose(linear(x, np.eye(5)), x)
    b = RNG.standard_normal(5)
    assert np.allclose(linear(x, np.eye(5), b), x + b)
    w = RNG.standard_normal((4, 5))
    row = np.array([sum(x[1, 2, kk] * w[j, kk] for kk in range(5)) for j in range(4)])
    assert np.allclose(linear(x, w)[1, 2], row)


def _pin_block_closed_forms(block):
    B, N, H, d = 2, 6, 2, 4
    C = H * d
    x, _, _, w_o, b_o = _case(B, N, H, d)
    # q = k = x, v = 0: the output is the proj bias
    w_qkv = np.concatenate([np.eye(C), np.eye(C), np.zeros((C, C))])
    y = block(x, w_qkv, None, w_o, b_o, H, d, 0.5, False)[0]
    assert np.allclose(y, np.broadcast_to(b_o, y.shape))
    # q = 0, v = x: uniform weights, the output is the key mean of x through the proj
    w_qkv = np.concatenate([np.zeros((C, C)), np.eye(C), np.eye(C)])
    y = block(x, w_qkv, None, w_o, b_o, H, d, 0.5, False)[0]
    mean = x.mean(axis=1, keepdims=True)
    assert np.allclose(y, np.broadcast_to(mean @ w_o.T + b_o, y.shape))


def test_split_puts_every_column_in_its_place():
    _pin_split(Bk.split_qkv)


def test_merge_undoes_the_split():
    _pin_merge(Bk.split_qkv, Bk.merge_heads)


def test_linear():
    _pin_linear(Bk.linear)


def test_block_closed_forms():
    _pin_block_closed_forms(Bk.attention_block_f64)


# ------------------------------------------------------------------ planted mistakes

def _split_heads_major(qkv, H, d):  # reads the columns as [H, 3, d] instead of [3, H, d]
    B, N, _ = qkv.shape
    r = qkv.reshape(B, N, H, 3, d)
    return tuple(np.ascontiguousarray(r[:, :, :, i].transpose(0, 2, 1, 3)) for i in range(3))


def _split_no_transpose(qkv, H, d):  # reshapes to [B, H, N, d] without moving the axes
    B, N, _ = qkv.shape
    r = qkv.reshape(B, N, 3, H * d)
    return tuple(r[:, :, i].reshape(B, H, N, d) for i in range(3))


def _merge_no_transpose(o):
    B, H, N, d = o.shape
    return o.reshape(B, N, H * d)


def _linear_untransposed(x, w, b=None):
    y = np.asarray(x) @ np.asarray(w)
    return y + b if b is not None else y


def _linear_no_bias(x, w, b=None):
    return np.asarray(x) @ np.asarray(w).T


@pytest.mark.parametrize("name", ["split_heads_major", "split_no_transpose", "merge_no_transpose",
                                  "linear_untransposed", "linear_no_bias"])
def test_pins_catch_planted_mistakes(monkeypatch, name):
    split, merge, lin = Bk.split_qkv, Bk.merge_heads, Bk.linear
    if name == "split_heads_major":
        split = _split_heads_major
    elif name == "split_no_transpose":
        split = _split_no_transpose
    elif name == "merge_no_transpose":
        merge = _merge_no_transpose
    elif name == "linear_untransposed":
        lin = _linear_untransposed
    else:
        lin = _linear_no_bias
    monkeypatch.setattr(Bk, "split_qkv", split)
    monkeypatch.setattr(Bk, "merge_heads", merge)
    monkeypatch.setattr(Bk, "linear", lin)
    caught = 0
    for pin in (lambda: _pin_split(Bk.split_qkv), lambda: _pin_merge(Bk.split_qkv, Bk.merge_heads),
                lambda: _pin_linear(Bk.linear),
                lambda: _pin_block_closed_forms(Bk.attention_block_f64)):
        try:
            pin()
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, name
