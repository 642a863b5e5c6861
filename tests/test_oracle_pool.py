"""The process-pool comparison used by the full-size parity tests, on the CPU.

A result that is the oracle's own output compares clean; one planted error is
found with its size and in its (batch, head) slice.  This checks the helper's
bookkeeping (slicing, worker dispatch, the reduction), not the kernel.
"""
import torch

import oracle
from seeded_inputs import make_qkv
from tests.oracle_pool import compare_all_slices


def test_pool_finds_a_planted_error_in_its_slice():
    q, k, v = make_qkv(2, 3, 300, 200, 64, "bf16", seed=3)
    o, lse = oracle.attention_f64(q, k, v, 0.125, True)
    o = torch.from_numpy(o)
    lse = torch.from_numpy(lse)
    eo, el, per = compare_all_slices(q, k, v, o, lse, 0.125, True, n_workers=2)
    assert len(per) == 6 and eo < 1e-12 and el < 1e-12
    o[1, 2, 5, 7] += 0.25
    lse[0, 1, 299] -= 0.5
    eo, el, per = compare_all_slices(q, k, v, o, lse, 0.125, True, n_workers=2)
    assert abs(eo - 0.25) < 1e-9 and abs(el - 0.5) < 1e-9
    worst_o = max(per, key=lambda r: r[1])
    worst_l = max(per, key=lambda r: r[2])
    assert worst_o[0] == 1 * 3 + 2 and worst_l[0] == 0 * 3 + 1
