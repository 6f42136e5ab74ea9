"""The split-K plan of the adapter products (lora_tc.cu), restated and checked
for what the kernel relies on.

A product of I x J output (128 x BN tiles, BN = J rounded up to 64, at most
128) over a reduction of Kred is cut into `splits` slices of kps (a multiple
of 64) per tile.  The slices of a tile form one thread-block cluster, which
exchanges partial tiles and meets at a cluster barrier, so:

- a tile's slices fit one portable cluster (at most 8 CTAs);
- every slice is non-empty and the slices cover the reduction;
- with more than one slice, every cluster of the launch is co-resident with
  the others (one wave: 8 GPCs, each holding floor(36 / splits) clusters at
  two CTAs per SM), and each slice runs at least four 64-deep steps;
- the LLaMA-7B shapes get one full wave of clusters for H and G.
"""

import itertools

import pytest

TBM, TBK = 128, 64
CTAS_PER_SM = 2
MAX_CLUSTER = 8


def ceil_div(a, b):
    return -(-a // b)


def tc_bn(J):
    return min(ceil_div(J, 64) * 64, 128)


def skinny_tiles(I, J):
    return max(1, ceil_div(I, TBM) * ceil_div(J, tc_bn(J)))


def coresident_clusters(z):
    return 8 * ((18 * CTAS_PER_SM) // z)


def plan_splits(tiles, Kred):
    Kred = max(Kred, 1)
    sp = 148 * CTAS_PER_SM // tiles
    sp = min(sp, max(Kred // (4 * TBK), 1), MAX_CLUSTER)
    while sp > 1 and tiles > coresident_clusters(sp):
        sp -= 1
    sp = max(sp, 1)
    kps = ceil_div(ceil_div(Kred, sp), TBK) * TBK
    return ceil_div(Kred, kps), kps


@pytest.mark.parametrize("I,J,Kred", list(itertools.product([16, 64, 128, 256, 4096, 11008], [8, 16, 64, 200],
                                                            [64, 256, 4096, 8192, 11008, 22016])))
def test_plan_invariants(I, J, Kred):
    tiles = skinny_tiles(I, J)
    splits, kps = plan_splits(tiles, Kred)
    assert 1 <= splits <= MAX_CLUSTER
    assert kps % TBK == 0 and kps > 0
    assert (splits - 1) * kps < Kred <= splits * kps   # every slice non-empty, the slices cover Kred
    if splits > 1:
        assert tiles <= coresident_clusters(splits)
        assert kps >= 4 * TBK


def test_pair_plan_shares_one_wave():
    """dB (I = N rows of the output, J = r) and dA (I = r, J = K) in one launch:
    their tiles add up, and the joint split still keeps every cluster co-resident."""
    for N, K, M, r in [(4096, 4096, 4096, 64), (11008, 4096, 4096, 64), (4096, 11008, 4096, 64),
                       (8192, 8192, 8192, 64), (22016, 8192, 8192, 64)]:
        tiles = skinny_tiles(N, r) + skinny_tiles(r, K)
        splits, kps = plan_splits(tiles, M)
        assert splits * tiles <= 148 * CTAS_PER_SM
        if splits > 1:
            assert tiles <= coresident_clusters(splits)


def test_llama7b_plans():
    """H = X A^T (M x r over K) and G = dY B (M x r over N) at M = 4096, r = 64:
    32 tiles of 128 x 64, eight slices each, which is exactly one wave of
    co-resident clusters of 8 (32 of them).  The joint dB + dA launch: 64 tiles
    in four slices for the q projection, 118 tiles in two for up and down."""
    tiles = skinny_tiles(4096, 64)
    assert tiles == 32 and coresident_clusters(8) == 32
    assert plan_splits(tiles, 4096) == (8, 512)
    assert plan_splits(tiles, 11008) == (8, 1408)
    assert plan_splits(skinny_tiles(4096, 64) + skinny_tiles(64, 4096), 4096) == (4, 1024)
    assert plan_splits(skinny_tiles(11008, 64) + skinny_tiles(64, 4096), 4096) == (2, 2048)
    assert plan_splits(skinny_tiles(4096, 64) + skinny_tiles(64, 11008), 4096) == (2, 2048)
