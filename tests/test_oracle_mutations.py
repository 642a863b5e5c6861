"""Plant mistakes in the oracle (on the CPU) and check that the pins notice.

Each mutation replaces one step of ``oracle.attention`` with a plausible
wrong version -- a dropped or inverted scale, an off-by-one or reversed
causal mask, softmax over the wrong axis, a wrong log base, a missing
normalisation, a shifted V index -- and requires that at least one of the
independent pins (closed forms and invariants, not brute force or torch)
fails.  This shows the pins are strong enough to trust the oracle.
"""
import numpy as np
import pytest

import oracle.attention as A
from tests import oracle_pins as P


def _scores_no_scale(q_rows, k, scale):
    return q_rows @ k.T


def _scores_divided(q_rows, k, scale):
    return (q_rows @ k.T) / scale


def _scores_reversed_keys(q_rows, k, scale):
    return scale * (q_rows @ k[::-1].T)


def _mask_strict(s, row_index):
    keys = np.arange(s.shape[1])[None, :]
    out = s.copy()
    out[keys >= row_index[:, None]] = -np.inf
    return out


def _mask_wrong_side(s, row_index):
    keys = np.arange(s.shape[1])[None, :]
    out = s.copy()
    out[keys < row_index[:, None]] = -np.inf
    return out


def _softmax_columns(s):
    m = np.max(s, axis=1)
    e = np.exp(s - m[:, None])
    e = np.where(np.isfinite(e), e, 0.0)
    colsum = e.sum(axis=0, keepdims=True)
    colsum = np.where(colsum > 0, colsum, 1.0)
    return e / colsum, m, e.sum(axis=1)


def _softmax_unnormalised(s):
    m = np.max(s, axis=1)
    e = np.exp(s - m[:, None])
    return e, m, e.sum(axis=1)


def _lse_no_max(m, l):
    return np.log(l)


def _lse_log2(m, l):
    return m + np.log2(l)


def _weighted_sum_shifted(p, v):
    return p @ np.roll(v, 1, axis=0)


MUTATIONS = {
    "scale_dropped": ("scores", _scores_no_scale),
    "scale_inverted": ("scores", _scores_divided),
    "keys_reversed": ("scores", _scores_reversed_keys),
    "causal_off_by_one": ("apply_causal_mask", _mask_strict),
    "causal_wrong_side": ("apply_causal_mask", _mask_wrong_side),
    "softmax_over_columns": ("softmax_rows", _softmax_columns),
    "softmax_not_normalised": ("softmax_rows", _softmax_unnormalised),
    "lse_without_max": ("logsumexp_rows", _lse_no_max),
    "lse_in_log2": ("logsumexp_rows", _lse_log2),
    "v_index_shifted": ("weighted_sum", _weighted_sum_shifted),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(A, attr, fn)
    failed = []
    with np.errstate(all="ignore"):
        for pin in P.INDEPENDENT_PINS:
            try:
                pin()
            except (AssertionError, ValueError, FloatingPointError):
                failed.append(pin.__name__)
    assert failed, f"mutation {name} passed every independent pin"
