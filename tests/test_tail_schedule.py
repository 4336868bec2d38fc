"""The tail split's schedule (sru::gemm::pair_next in csrc/sru_gemm.cuh), restated
on the host: with T = F P + R output tiles on P CTA pairs, pair p takes whole tiles
p + i P for i < F; then pair p < R the long k-piece of tail tile F P + p, and pair
p >= R the short pieces of tail tiles F P + (p - R) + j (P - R) below F P + R.
Every tail tile must get exactly one long and one short piece (two addends onto
zero: the deterministic sum), every whole tile exactly one unit, and no pair more
than q = ceil(R / (P - R)) short pieces."""
import math

import pytest


def _schedule(tiles, P):
    F, R = tiles // P, tiles % P
    units = {}
    for p in range(P):
        i = 0
        while True:
            if i < F:
                kind, tile = "whole", p + i * P
            elif p < R:
                if i != F:
                    break
                kind, tile = "long", F * P + p
            else:
                t = (p - R) + (i - F) * (P - R)
                if t >= R:
                    break
                kind, tile = "short", F * P + t
            units.setdefault(p, []).append((kind, tile))
            i += 1
    return F, R, units


@pytest.mark.parametrize("P", [74, 66, 57])
def test_every_tile_is_covered_once_per_piece(P):
    for tiles in range(P + 1, 4 * P):
        F, R, units = _schedule(tiles, P)
        if R == 0:
            continue
        seen = {}
        for p, us in units.items():
            for kind, tile in us:
                seen.setdefault(tile, []).append(kind)
        for t in range(F * P):
            assert seen[t] == ["whole"], (tiles, t)
        for t in range(F * P, tiles):
            assert sorted(seen[t]) == ["long", "short"], (tiles, t, seen.get(t))
        q = math.ceil(R / (P - R))
        assert max(sum(k == "short" for k, _ in us) for us in units.values()) == q


def test_split_used_by_the_host_costs_at_most_two_thirds_of_a_round():
    # the host splits for q <= 2 only: s = K / (q + 1), so every pair's tail work
    # (one long piece, or q short ones) is at most q / (q + 1) <= 2/3 of a tile
    for R in range(1, 74):
        q = math.ceil(R / (74 - R))
        if q <= 2:
            assert max(1 - 1 / (q + 1), q / (q + 1)) <= 2 / 3 + 1e-12
