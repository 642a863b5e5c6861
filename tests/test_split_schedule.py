"""The split-mode work division, replayed on the CPU.

A consistency check of restated formulas (it calls no kernel): the kernel's
WorkCursor gives CTA c the flattened (unit, key tile) steps
[c * S / G, (c + 1) * S / G), where a unit is one query pair of one head with
the key tiles its queries see (all nk, or under the causal mask min(nk, i + 1)
for its later query tile i).  It locates a step's unit with a closed-form
prefix sum per head, m (m + 1) + (qp - m) nk with m = min(qp, nk / 2), and its
inverse through a square root, and derives each piece's index, the piece
count and the CTA of piece 0 from "CTAs c >= 1 whose range begins at or
before step x".  This test replays that arithmetic for many shapes and grids
and checks it against direct enumeration: the closed forms agree with the
running sums, every step is covered exactly once, piece k of a unit is
processed by CTA c_first + k, and no CTA uses a workspace slot twice.
"""
import itertools
import math

import pytest


class Shape:
    def __init__(self, heads, q_tiles, nk, causal):
        self.heads, self.q_tiles, self.nk, self.causal = heads, q_tiles, nk, causal
        self.pairs = -(-q_tiles // 2)
        self.per_head = sum(self.steps(qp) for qp in range(self.pairs))
        self.S = heads * self.per_head

    def steps(self, qp):  # split_unit_steps
        if not self.causal:
            return self.nk
        last = 2 * qp + 1 if 2 * qp + 1 < self.q_tiles else 2 * qp
        return min(self.nk, last + 1)

    def prefix(self, qp):  # split_head_prefix (closed form)
        if not self.causal:
            return qp * self.nk
        m = min(qp, self.nk // 2)
        return m * (m + 1) + (qp - m) * self.nk

    def locate_pair(self, rem):  # split_locate_pair (square root, then corrected)
        if not self.causal:
            qp = rem // self.nk
        else:
            a = self.nk // 2
            if rem < a * (a + 1):
                m = int((math.sqrt(4.0 * rem + 1.0) - 1.0) * 0.5)
                while m > 0 and m * (m + 1) > rem:
                    m -= 1
                while (m + 1) * (m + 2) <= rem:
                    m += 1
                qp = m
            else:
                qp = a + (rem - a * (a + 1)) // self.nk
        return min(qp, self.pairs - 1)

    def unit_start(self, u):
        bh, qp = divmod(u, self.pairs)
        return bh * self.per_head + self.prefix(qp)

    def locate_unit(self, step):
        bh, rem = divmod(step, self.per_head)
        return bh * self.pairs + self.locate_pair(rem)


def starts_le(S, G, x):
    c = ((x + 1) * G - 1) // S
    return min(c, G - 1)


def cursor_items(sh, G, cta):
    """Items (unit, j0, j1, piece, pieces, c_first) of one CTA, as the kernel forms them."""
    S = sh.S
    begin, end = S * cta // G, S * (cta + 1) // G
    if begin >= end:
        return []
    u = sh.locate_unit(begin)
    j_first = begin - sh.unit_start(u)
    u_last = sh.locate_unit(end - 1)
    j_end = end - sh.unit_start(u_last)

    def pieces_of(uu, j0):
        a = sh.unit_start(uu)
        ca = starts_le(S, G, a)
        return (starts_le(S, G, a + j0) - ca, 1 + starts_le(S, G, a + sh.steps(uu % sh.pairs) - 1) - ca,
                ca)

    out = []
    for uu in range(u, u_last + 1):
        j0 = j_first if uu == u else 0
        j1 = j_end if uu == u_last else sh.steps(uu % sh.pairs)
        if uu == u:
            piece, pieces, c_first = pieces_of(uu, j_first)
        elif uu == u_last:
            piece, pieces, c_first = pieces_of(uu, 0)
        else:
            piece, pieces, c_first = 0, 1, cta
        out.append((uu, j0, j1, piece, pieces, c_first))
    return out


def check(sh, G):
    S = sh.S
    G = min(G, S)
    # closed forms against running sums
    run = 0
    for qp in range(sh.pairs):
        assert sh.prefix(qp) == run
        for r in range(run, run + sh.steps(qp)):
            assert sh.locate_pair(r) == qp
        run += sh.steps(qp)
    assert run == sh.per_head
    covered = {}
    pieces_seen = {}
    for c in range(G):
        slots = set()
        for (u, j0, j1, piece, pieces, c_first) in cursor_items(sh, G, c):
            assert 0 <= j0 < j1 <= sh.steps(u % sh.pairs)
            for j in range(j0, j1):
                assert (u, j) not in covered
                covered[(u, j)] = c
            if pieces > 1:
                assert c == c_first + piece
                slot = 1 if piece == 0 else 0
                assert slot not in slots
                slots.add(slot)
                pieces_seen.setdefault(u, set()).add(piece)
    assert len(covered) == S
    for u in range(sh.heads * sh.pairs):
        ctas = sorted({covered[(u, j)] for j in range(sh.steps(u % sh.pairs))})
        if len(ctas) > 1:
            assert pieces_seen[u] == set(range(len(ctas)))
            assert ctas == list(range(ctas[0], ctas[0] + len(ctas)))
    sizes = [S * (c + 1) // G - S * c // G for c in range(G)]
    assert max(sizes) - min(sizes) <= 1


CASES = [(1, 4, 4, 8), (2, 4, 4, 16), (32, 26, 13, 148), (32, 26, 13, 100), (1, 16, 16, 128),
         (1, 5, 7, 5), (1, 1, 1, 1), (1, 2, 50, 148), (7, 6, 3, 20), (64, 50, 50, 148),
         (64, 13, 13, 148)]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("heads,q_tiles,nk,G", CASES)
def test_split_cover_and_pieces(heads, q_tiles, nk, G, causal):
    check(Shape(heads, q_tiles, nk, causal), G)


def test_exhaustive_small():
    for heads, q_tiles, nk, causal in itertools.product(range(1, 4), range(1, 8), range(1, 8),
                                                        (False, True)):
        sh = Shape(heads, q_tiles, nk, causal)
        for G in range(1, min(sh.S, 40) + 1):
            check(sh, G)


def test_locate_large_causal_heads():
    """The square-root inverse at long-context sizes (256 query tiles, 256 key tiles)."""
    sh = Shape(1, 256, 256, True)
    run = 0
    for qp in range(sh.pairs):
        for r in (run, run + sh.steps(qp) - 1):
            assert sh.locate_pair(r) == qp
        run += sh.steps(qp)
