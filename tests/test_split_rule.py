"""attn_plan's split/unit decision against the documented rule, restated independently.

Split mode is chosen for non-causal problems when unit mode leaves the grid
ragged (fewer units than SMs, or a last wave under 90 % full) and the serial
key-tile steps it saves per CTA exceed its cost of merging pieces: about
3.5 + 0.56 steps per piece at d = 64 and 2.5 + 1.03 at d = 128.  Unit mode
counts dual units (odd query-tile count, two or more heads); split mode shares
out plain units (B * H * ceil(q_tiles / 2)).
"""
import itertools

import pytest

import exact_attention_153_b200 as A


def rule(B, H, Nq, Nk, d, causal, sms):
    q_tiles = -(-Nq // 128)
    kv = -(-Nk // 128)
    bh = B * H
    if causal:
        return False
    dual = q_tiles % 2 == 1 and bh >= 2
    units = bh * (q_tiles // 2 if dual else -(-q_tiles // 2)) + ((bh + 1) // 2 if dual else 0)
    steps = bh * (-(-q_tiles // 2)) * kv
    if steps < 2:
        return False
    grid = min(units, sms)
    waves = -(-units // grid)
    if units / (grid * waves) >= 0.9 and units >= sms:
        return False
    grid_s = min(steps, sms)
    pieces = -(-kv * grid_s // steps)
    cost = 3.5 + 0.56 * pieces if d == 64 else 2.5 + 1.03 * pieces
    return waves * kv - (-(-steps // grid_s)) > cost


SHAPES = list(itertools.product([1, 2, 16], [1, 3, 4], [100, 400, 1600, 2000, 6400],
                                [400, 2000, 8192], [64, 128], [0, 1]))


@pytest.mark.parametrize("B,H,Nq,Nk,d,causal", SHAPES)
def test_split_decision_matches_the_rule(B, H, Nq, Nk, d, causal):
    for sms in (148, 132):
        p = A.attn_plan(B, H, Nq, Nk, d, causal, sms)
        assert bool(p["split"]) == rule(B, H, Nq, Nk, d, causal, sms), (B, H, Nq, Nk, d, causal, sms)
        assert (p["workspace_bytes"] > 0) == bool(p["split"])
