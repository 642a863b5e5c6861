"""The split-mode work division, replayed on the CPU.

The kernel's WorkCursor gives CTA c the flattened (unit, key tile) steps
[c * S / G, (c + 1) * S / G) and derives, for a unit cut into pieces, each
piece's index, the piece count and the CTA of piece 0 from one closed form
("CTAs c >= 1 whose range begins at or before step x").  This test replays
that arithmetic for many (units, key tiles, grid) combinations and checks it
against direct enumeration: every step is covered exactly once, piece k of a
unit is processed by CTA c_first + k, and no CTA uses a workspace slot twice.
"""
import itertools

import pytest


def starts_le(S, G, x):
    c = ((x + 1) * G - 1) // S
    return min(c, G - 1)


def cursor_items(units, nk, G, cta):
    """Items (unit, j0, j1, piece, pieces, c_first) of one CTA, as the kernel forms them."""
    S = units * nk
    idx, end = S * cta // G, S * (cta + 1) // G
    out = []
    while idx < end:
        u, j0 = divmod(idx, nk)
        j1 = min(nk, j0 + (end - idx))
        a = u * nk
        ca = starts_le(S, G, a)
        piece = starts_le(S, G, a + j0) - ca
        pieces = 1 + starts_le(S, G, a + nk - 1) - ca
        out.append((u, j0, j1, piece, pieces, ca))
        idx += j1 - j0
    return out


CASES = [(2, 4, 8), (4, 4, 16), (448, 13, 148), (448, 13, 100), (8, 16, 128), (3, 7, 5),
         (1, 1, 1), (1, 50, 148), (7, 3, 20), (1600, 50, 148), (64, 13, 148)]


@pytest.mark.parametrize("units,nk,G", CASES)
def test_split_cover_and_pieces(units, nk, G):
    S = units * nk
    G = min(G, S)
    covered = {}
    pieces_seen = {}
    for c in range(G):
        slots = set()
        for (u, j0, j1, piece, pieces, c_first) in cursor_items(units, nk, G, c):
            for j in range(j0, j1):
                assert (u, j) not in covered
                covered[(u, j)] = c
            if pieces > 1:
                assert c == c_first + piece
                slot = 1 if piece == 0 else 0
                assert slot not in slots
                slots.add(slot)
                pieces_seen.setdefault(u, set()).add(piece)
                assert (pieces, c_first) == (pieces, c_first)
    assert len(covered) == S
    for u in range(units):
        ctas = sorted({covered[(u, j)] for j in range(nk)})
        expected = len(ctas)
        if expected > 1:
            assert pieces_seen[u] == set(range(expected))
            assert ctas == list(range(ctas[0], ctas[0] + expected))
    # every CTA gets floor or ceil of S / G steps
    sizes = [S * (c + 1) // G - S * c // G for c in range(G)]
    assert max(sizes) - min(sizes) <= 1


def test_exhaustive_small():
    for units, nk, G in itertools.product(range(1, 7), range(1, 7), range(1, 40)):
        if G > units * nk:
            continue
        test_split_cover_and_pieces(units, nk, G)
