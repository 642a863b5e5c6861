"""CPU tests of the float64 oracle against its pins (no GPU)."""
import numpy as np
import torch
import pytest

import oracle.attention as A
from seeded_inputs import WORKLOADS, make_qkv, workload
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_row_block_size_does_not_matter():
    """Blocking the materialised S by rows is not a reordering of any sum."""
    q, k, v = make_qkv(1, 2, 300, 300, 64, "fp16", 7)
    o1, l1 = A.attention_f64(q, k, v, 0.125, True, row_block=300)
    o2, l2 = A.attention_f64(q, k, v, 0.125, True, row_block=37)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_head_rows_matches_full():
    """The per-row entry used for sampled parity equals the full oracle."""
    q, k, v = make_qkv(2, 2, 200, 150, 32, "bf16", 8)
    o, lse = A.attention_f64(q, k, v, 0.2, True)
    rows = np.array([0, 5, 149, 150, 199])
    oh, lh = A.attention_head_rows(q[1, 0, rows], k[1, 0], v[1, 0], 0.2, True, rows)
    assert np.array_equal(oh, o[1, 0, rows]) and np.array_equal(lh, lse[1, 0, rows])


def test_exact_upcast():
    """fp16 / bf16 inputs reach the oracle unchanged (exact upcast)."""
    q, _, _ = make_qkv(1, 1, 4, 4, 8, "bf16", 9)
    assert np.array_equal(A.to_f64(q), q.double().numpy())


def test_workload_inputs_are_deterministic():
    w = workload(0)
    a = make_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, w.seed)
    b = make_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, w.seed)
    for x, y in zip(a, b):
        assert x.dtype == y.dtype and torch.equal(x, y)


def test_workload_table():
    """Shapes of the five workloads (the pages' YOLO, LLM and long-context shapes)."""
    shapes = [(w.B, w.H, w.Nq, w.d, w.dtype, w.causal) for w in WORKLOADS]
    assert shapes == [(1, 2, 400, 64, "fp16", False), (16, 4, 1600, 64, "fp16", False),
                      (16, 4, 6400, 64, "bf16", False), (32, 16, 2048, 64, "fp16", True),
                      (1, 32, 32768, 128, "bf16", True)]
    assert WORKLOADS[4].qk_scale == 0.5


def test_small_workload_oracle_runs():
    """The 20x20 YOLO workload finishes in the oracle and gives finite results."""
    w = workload(0)
    q, k, v = make_qkv(w.B, w.H, w.Nq, w.Nk, w.d, w.dtype, w.seed)
    o, lse = A.attention_f64(q, k, v, w.scale, w.causal)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert o.shape == (1, 2, 400, 64) and lse.shape == (1, 2, 400)
