"""attn_plan's split/unit decision against the documented rule, restated independently.

A consistency check of a restated host formula (it calls no kernel): split
mode is chosen when unit mode leaves the grid ragged (fewer units than SMs,
or a last wave under 90 % full) and the serial key-tile steps it saves per
CTA exceed its cost of merging pieces: about 3.5 + 0.56 steps per piece at
d = 64 and 2.5 + 1.03 at d = 128, 1.3 times that under the causal mask.
Unit mode counts dual units (odd
query-tile count, two or more heads, non-causal) and, under the causal mask,
units of a heavy query pair plus its light mirror; split mode shares out
plain units (one query pair of one head), each with the key tiles its later
query tile sees (min(nk, i + 1) for query tile i under the causal mask).
"""
import itertools

import pytest

import exact_attention_153_b200 as A


def pair_steps(qp, q_tiles, kv, causal):
    if not causal:
        return kv
    last = 2 * qp + 1 if 2 * qp + 1 < q_tiles else 2 * qp
    return min(kv, last + 1)


def rule(B, H, Nq, Nk, d, causal, sms):
    q_tiles = -(-Nq // 128)
    kv = -(-Nk // 128)
    pairs = -(-q_tiles // 2)
    bh = B * H
    dual = (not causal) and q_tiles % 2 == 1 and bh >= 2
    if causal:
        per_head = (pairs + 1) // 2
        units = bh * per_head
        unit_steps = max(pair_steps(pairs - 1 - b, q_tiles, kv, 1) +
                         (pair_steps(b, q_tiles, kv, 1) if pairs - 1 - b != b else 0)
                         for b in range(per_head))
    else:
        units = bh * (q_tiles // 2 if dual else pairs) + ((bh + 1) // 2 if dual else 0)
        unit_steps = kv
    per_pair = [pair_steps(qp, q_tiles, kv, causal) for qp in range(pairs)]
    steps = bh * sum(per_pair)
    if steps < 2:
        return False
    grid = min(units, sms)
    waves = -(-units // grid)
    if units / (grid * waves) >= 0.9 and units >= sms:
        return False
    grid_s = min(steps, sms)
    pieces = -(-max(per_pair) * grid_s // steps)
    cost = (3.5 + 0.56 * pieces if d == 64 else 2.5 + 1.03 * pieces) * (1.3 if causal else 1.0)
    return waves * unit_steps - (-(-steps // grid_s)) > cost


SHAPES = list(itertools.product([1, 2, 16], [1, 3, 4], [100, 400, 1600, 2000, 6400],
                                [400, 2000, 8192], [64, 128], [0, 1]))


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", SHAPES)
def test_split_decision_matches_the_rule(B, H, Nq, Nk, d, causal):
    for sms in (148, 132):
        p = A.attn_plan(B, H, Nq, Nk, d, causal, sms)
        assert bool(p["split"]) == rule(B, H, Nq, Nk, d, causal, sms), (B, H, Nq, Nk, d, causal, sms)
        assert (p["workspace_bytes"] > 0) == bool(p["split"])
        q_tiles, kv = -(-Nq // 128), -(-Nk // 128)
        assert p["split_steps"] == B * H * sum(pair_steps(qp, q_tiles, kv, causal)
                                               for qp in range(-(-q_tiles // 2)))
