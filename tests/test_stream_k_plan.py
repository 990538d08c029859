"""Bookkeeping of the stream-K split of the prefill GEMM, restated on the CPU.

The kernel cuts the U = tiles x k-blocks units into ranges [U c / G, U (c+1) / G)
per CTA c and walks them tile by tile; a piece of a split tile goes to slot 2c
(the CTA's first piece) or 2c + 1 (its last). The fix-up kernel finds the CTAs
covering tile t with owner(u) = ceil((u + 1) G / U) - 1 and reads slot 2c when
c's range starts inside the tile, else 2c + 1. These tests check that the two
rules agree: every piece written is read exactly once, and no CTA writes more
than two pieces or writes one slot twice."""
import random


def ranges(U, G):
    return [U * c // G for c in range(G + 1)]


def owner(u, U, G):
    return ((u + 1) * G + U - 1) // U - 1


def kernel_pieces(U, G, nkb):
    """(tile -> slots written) from the per-CTA walk of the kernel."""
    ub = ranges(U, G)
    written = {}
    for c in range(G):
        u, seg, slots = ub[c], 0, []
        while u < ub[c + 1]:
            t = u // nkb
            kb0 = u - t * nkb
            kb1 = min(nkb, kb0 + ub[c + 1] - u)
            if not (kb0 == 0 and kb1 == nkb):
                slot = 2 * c + (0 if seg == 0 else 1)
                slots.append(slot)
                written.setdefault(t, []).append(slot)
            u += kb1 - kb0
            seg += 1
        assert len(slots) == len(set(slots)) <= 2
    return written


def fixup_reads(U, G, nkb, tiles):
    ub = ranges(U, G)
    reads = {}
    for t in range(tiles):
        cf, cl = owner(t * nkb, U, G), owner(t * nkb + nkb - 1, U, G)
        if cf == cl:
            continue
        reads[t] = [2 * c + (0 if ub[c] >= t * nkb else 1) for c in range(cf, cl + 1)]
    return reads


def test_owner_finds_the_range_holding_each_unit():
    rng = random.Random(1)
    for _ in range(300):
        U = rng.randint(1, 20000)
        G = rng.randint(1, min(U, 148))
        ub = ranges(U, G)
        for u in rng.sample(range(U), min(U, 40)):
            c = owner(u, U, G)
            assert ub[c] <= u < ub[c + 1]


def test_pieces_written_are_the_pieces_read():
    rng = random.Random(2)
    shapes = [(40, 54), (160, 54), (320, 54), (6, 32), (30, 33), (1, 64), (148, 20), (149, 40)]
    shapes += [(rng.randint(1, 400), rng.randint(1, 80)) for _ in range(200)]
    for tiles, nkb in shapes:
        U = tiles * nkb
        G = min(148, U)  # the launch never gives a CTA an empty range
        written = kernel_pieces(U, G, nkb)
        reads = fixup_reads(U, G, nkb, tiles)
        assert set(written) == set(reads)
        for t in written:
            assert sorted(written[t]) == sorted(reads[t]), (tiles, nkb, t)
            assert len(written[t]) >= 2
