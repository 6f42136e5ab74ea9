"""The stream-K partition of the fused GEMM's shared tiles, as the pair kernel
computes it (unit u of U takes tail steps [u S / U, (u+1) S / U); the unit
holding step g is ((g+1) U - 1) / S), with the invariants the kernel's piece
bookkeeping relies on:

- every K-step of the shared tiles belongs to exactly one unit, and the
  inverse formula finds it;
- a tile's pieces come from consecutive units, at most ceil(ns / share) + 1;
- a unit's piece in a shared tile is its first segment exactly when the unit
  starts inside that tile (the finisher's rule for which of the unit's two
  piece slots to read), and only a unit's first or last segment can be a
  partial piece (its middle segments cover whole tiles);
- the host's split decision: units never take fewer than 16 K-steps; the
  default mode keeps the LLaMA-7B tiles of 17 and 65 K-steps whole, splits the
  last round of the 173-step tiles (the 11008-long reductions: down forward,
  up dgrad, measured 0-1.5 % faster split) and a single round of few long tiles.
"""

import itertools

import pytest

SK_MIN_STEPS = 16      # fewest K-steps a unit takes
SK_COST_STEPS = 33     # a split cluster's extra cost, in K-steps
TILE_COST_STEPS = 8    # a whole tile's fill and drain, in K-steps


def sk_begin(steps, units, u):
    return u * steps // units


def sk_unit_of(steps, units, g):
    return ((g + 1) * units - 1) // steps


def plan(tiles, slots, ns):
    """(tail tiles, units, split by the default mode) as the launch computes them."""
    tail = tiles % slots
    steps = tail * ns
    units = min(slots, max(1, steps // SK_MIN_STEPS))
    split = tail > 0 and -(-steps // units) + SK_COST_STEPS < ns + TILE_COST_STEPS
    return tail, units, split


SHAPES = list(itertools.product([1, 5, 8, 16, 32, 54, 73, 128, 344], [74, 72, 80], [2, 9, 17, 33, 65, 173]))


@pytest.mark.parametrize("tiles,slots,ns", SHAPES)
def test_partition_invariants(tiles, slots, ns):
    tail, units, _ = plan(tiles, slots, ns)
    if tail == 0:
        return
    steps = tail * ns
    owner = [None] * steps
    for u in range(units):
        lo, hi = sk_begin(steps, units, u), sk_begin(steps, units, u + 1)
        assert lo < hi, "every unit has work"
        assert hi - lo >= min(SK_MIN_STEPS, steps // units)
        for g in range(lo, hi):
            assert owner[g] is None
            owner[g] = u
            assert sk_unit_of(steps, units, g) == u
    assert None not in owner
    share = steps // units
    for t in range(tail):
        first, last = sk_unit_of(steps, units, t * ns), sk_unit_of(steps, units, (t + 1) * ns - 1)
        pieces = list(range(first, last + 1))
        assert all(owner[g] in pieces for g in range(t * ns, (t + 1) * ns))
        assert len(pieces) <= -(-ns // share) + 1
        if len(pieces) == 1:
            continue
        for u in pieces:
            lo, hi = sk_begin(steps, units, u), sk_begin(steps, units, u + 1)
            starts_inside = lo >= t * ns
            first_tile, last_tile = lo // ns, (hi - 1) // ns
            if starts_inside:
                assert first_tile == t        # slot 0: the unit's first segment
            else:
                assert last_tile == t and first_tile < t   # slot 1: its last segment


def test_default_mode_choices():
    # LLaMA-7B projections, 74 cluster slots: 128 tiles of 65 or 17 steps, 344 of 65 -> whole tiles
    for tiles, ns in ((128, 65), (128, 17), (344, 65)):
        assert not plan(tiles, 74, ns)[2], (tiles, ns)
    # 128 tiles of 173 steps: the 54 of the last round go to 74 units of ~127 steps
    assert plan(128, 74, 173) == (54, 74, True)
    # 8 tiles of 65 steps: 32 units of ~16 steps beat one round of whole tiles
    tail, units, split = plan(8, 74, 65)
    assert (tail, units, split) == (8, 32, True)
