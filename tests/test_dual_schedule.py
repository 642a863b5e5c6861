"""The unit-mode work division with dual units, replayed on the CPU.

With an odd number of 128-row query tiles per (batch, head), unit mode keeps
the full query-tile pairs of every head as ordinary units and pairs the lone
last tiles of heads 2d and 2d + 1 in dual units placed after them (the last
one alone when the head count is odd).  This test replays that decoding for
many shapes and checks that every (batch * head, query tile) is computed
exactly once, that both tiles of an ordinary unit share one head and one
key stream, and that the unit counts match attn_plan.
"""
import itertools

import pytest

import exact_attention_153_b200 as A


def decode(BH, q_tiles):
    """Units as the kernel forms them: list of [(bh, q_tile), ...] per unit."""
    dual = q_tiles % 2 == 1 and BH >= 2
    uph = q_tiles // 2 if dual else (q_tiles + 1) // 2
    units = []
    for bh in range(BH):
        for qp in range(uph):
            tiles = [(bh, 2 * qp)]
            if 2 * qp + 1 < q_tiles:
                tiles.append((bh, 2 * qp + 1))
            units.append(tiles)
    if dual:
        for d in range((BH + 1) // 2):
            h0 = 2 * d
            tiles = [(h0, q_tiles - 1)]
            if h0 + 1 < BH:
                tiles.append((h0 + 1, q_tiles - 1))
            units.append(tiles)
    return units, (BH + 1) // 2 if dual else 0


@pytest.mark.parametrize("B,H,Nq", list(itertools.product([1, 2, 3], [1, 2, 5], [100, 128, 129, 300, 1600, 1700])))
def test_every_query_tile_once(B, H, Nq):
    BH = B * H
    q_tiles = -(-Nq // 128)
    units, n_dual = decode(BH, q_tiles)
    seen = [t for u in units for t in u]
    assert sorted(seen) == [(bh, qt) for bh in range(BH) for qt in range(q_tiles)]
    for u in units[:len(units) - n_dual]:
        assert len({bh for bh, _ in u}) == 1  # ordinary units share one head
    p = A.attn_plan(B, H, Nq, Nq, 64, 0, 148)
    assert p["num_units"] == len(units) and p["dual_units"] == n_dual
    # a dual unit never idles a warpgroup except the last one of an odd head count
    for u in units[len(units) - n_dual:-1]:
        assert len(u) == 2


def test_causal_has_no_dual_units():
    for Nq in (300, 1700):
        assert A.attn_plan(2, 3, Nq, Nq, 64, 1, 148)["dual_units"] == 0
