"""Host model of the serving kernels' work split (stream-K) and partial-tile bookkeeping.

Every serving kernel orders the chunks of all tiles of all operands of a launch into one
sequence of `total` chunks and gives unit u of G units (a warp, or a CTA for the
tensor-memory kernels) the contiguous range [u*total/G, (u+1)*total/G). A tile whose chunks
[a, b) span several units is summed through the workspace: each unit that holds a piece of it
writes a partial tile into slot 1 if that piece is the unit's last and the unit began before
the tile, else slot 0; an atomic ticket keyed by the tile's first unit c1 counts the pieces,
and the unit that sees the count reach c2 - c1 adds the pieces of units c1..c2 in order. These
tests restate those integer formulas (as written in kernels_spl.cuh and kernels_umma.cuh) and
check, exhaustively over small sizes, the invariants the kernels rely on."""
import itertools

import pytest


def unit_range(u, G, total):
    return u * total // G, (u + 1) * total // G


def first_last_units(a, b, G, total):
    # the unit holding chunk a, and the unit holding chunk b - 1
    return ((a + 1) * G - 1) // total, (b * G - 1) // total


def slot_of(u, c1, a, G, total):
    lo1 = c1 * total // G
    return 1 if (u == c1 and lo1 < a) else 0


def pieces(tiles_nch, G):
    """(tile, unit, slot) of every piece of every tile split between units."""
    total = sum(tiles_nch)
    G = min(G, total)
    out, begin = [], 0
    for t, nch in enumerate(tiles_nch):
        a, b = begin, begin + nch
        begin = b
        c1, c2 = first_last_units(a, b, G, total)
        if c1 == c2:
            continue
        for u in range(c1, c2 + 1):
            out.append((t, u, slot_of(u, c1, a, G, total), c1, c2))
    return out, total, G


CASES = [tiles for n in range(1, 6) for tiles in itertools.product([1, 2, 3, 5, 8], repeat=n)]


@pytest.mark.parametrize("G", [1, 2, 3, 4, 7, 16])
def test_every_chunk_belongs_to_exactly_one_unit(G):
    for tiles in CASES:
        total = sum(tiles)
        g = min(G, total)
        owners = [None] * total
        for u in range(g):
            lo, hi = unit_range(u, g, total)
            assert hi > lo  # no unit is empty once G <= total
            for c in range(lo, hi):
                assert owners[c] is None
                owners[c] = u
        assert all(o is not None for o in owners)
        # the closed forms name the owners of a tile's first and last chunk
        begin = 0
        for nch in tiles:
            a, b = begin, begin + nch
            begin = b
            c1, c2 = first_last_units(a, b, g, total)
            assert owners[a] == c1 and owners[b - 1] == c2


@pytest.mark.parametrize("G", [2, 3, 4, 7, 16])
def test_partial_slots_never_collide_and_the_reader_finds_them(G):
    for tiles in CASES:
        ps, total, g = pieces(tiles, G)
        used = {}
        for t, u, slot, c1, c2 in ps:
            assert (u, slot) not in used, (tiles, G, t, u, slot, used.get((u, slot)))
            used[(u, slot)] = t
        # the last arriver of tile t reads, for q = c1..c2, slot (q == c1 and lo1 < a): exactly
        # the slots the pieces were written to
        by_tile = {}
        for t, u, slot, c1, c2 in ps:
            by_tile.setdefault(t, []).append((u, slot, c1, c2))
        begin = 0
        for t, nch in enumerate(tiles):
            a, b = begin, begin + nch
            begin = b
            if t not in by_tile:
                continue
            written = {(u, s) for u, s, _, _ in by_tile[t]}
            c1, c2 = by_tile[t][0][2], by_tile[t][0][3]
            read = {(q, slot_of(q, c1, a, g, total)) for q in range(c1, c2 + 1)}
            assert read == written
            # the ticket counts one arrival per piece; the arrival that sees c2 - c1 is the last
            assert len(by_tile[t]) == c2 - c1 + 1


def test_a_unit_holds_at_most_two_split_pieces():
    for G in (2, 3, 5, 16):
        for tiles in CASES:
            ps, _, _ = pieces(tiles, G)
            per_unit = {}
            for t, u, slot, _, _ in ps:
                per_unit.setdefault(u, set()).add(t)
            assert all(len(v) <= 2 for v in per_unit.values())


def test_tickets_are_keyed_by_distinct_first_units():
    """Two split tiles never share their first unit c1, so one ticket word per unit suffices
    (the workspace holds one per warp of the largest grid)."""
    for G in (2, 3, 5, 16):
        for tiles in CASES:
            ps, _, _ = pieces(tiles, G)
            firsts = {}
            for t, u, slot, c1, c2 in ps:
                firsts.setdefault(c1, set()).add(t)
            assert all(len(v) == 1 for v in firsts.values())
