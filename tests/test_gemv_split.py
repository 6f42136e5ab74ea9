"""The work split of the few-token forward (gemv.cu), restated and checked for
the invariants its piece bookkeeping relies on.

The weight is cut into units (16-row tile t, 256-wide K step s; unit t S + s,
S = ceil(K / 256)).  CTA c takes [start(c), start(c+1)): an even split of
U + P pc + JT hc units of work, where each of the first P = min(JT S, G) CTAs
(an H part each) gives up pc units and each of the first JT CTAs (adding a
tile of H) gives up hc.  Warp w of a CTA with range [a, a + L) starts at
a + floor(w L / 8).  A warp stores one fp32 piece per tile it touches, in its
CTA's slot (t - ta) + w (ta: the CTA's first tile).  The workspace has SLOTS
slots per CTA, sized for the longest range at one CTA per SM.  The checks:

- the CTA starts run from 0 to U without decreasing, and the warp ranges
  partition each CTA range;
- the inverse lookups the tile finish uses (the CTA whose range holds a unit,
  by binary search over the starts; the warp whose range holds it, by a
  closed form) find the range that holds the unit;
- every (CTA, slot) a piece goes to is inside the workspace and taken by one
  (warp, tile) only;
- the warp that finishes a tile (the one holding its last unit) sits in the
  last CTA on the tile, and every earlier piece of the tile is in that CTA or
  an earlier one.
"""

import itertools

import pytest

WARPS = 8          # warps per CTA
PC, HC = 1, 3      # default weight units given up for an H part / for adding a tile of H
SMS = 148          # B200


def ceil_div(a, b):
    return -(-a // b)


def layout(N, K, r, sms=SMS, ctas_per_sm=2):
    """Tiles, K steps, units, adapter tiles and slots per CTA as gemv_layout sizes them."""
    T = ceil_div(N, 16)
    S = ceil_div(K // 64, 4)
    U = T * S
    JT = ceil_div(r, 16)
    g_min = sms
    maxlen = ceil_div(U + JT * (HC + S // 16), g_min) + PC
    slots = ceil_div(maxlen, S) + 1 + (WARPS - 1)
    return dict(T=T, S=S, U=U, JT=JT, HP=JT * S, SLOTS=slots, G_max=ctas_per_sm * sms)


def cta_start(c, U, G, P, pc, JT, hc):
    total = U + P * pc + JT * hc
    return c * total // G - min(c, P) * pc - min(c, JT) * hc


def warp_start(a, L, w):
    return a + ((w * L) >> 3)


def warp_owner(a, L, u):
    return ((u - a + 1) * WARPS - 1) // L


def cta_owner(starts, G, u):
    lo, hi = 0, G - 1
    while lo < hi:
        mid = (lo + hi + 1) >> 1
        if starts[mid] <= u:
            lo = mid
        else:
            hi = mid - 1
    return lo


SHAPES = list(itertools.product([16, 100, 4096, 11008], [64, 512, 4096, 11008], [8, 64, 256], [SMS, 2 * SMS]))


@pytest.mark.parametrize("N,K,r,G", SHAPES)
def test_split_invariants(N, K, r, G):
    L_ = layout(N, K, r)
    S, U, JT, HP, SLOTS = L_["S"], L_["U"], L_["JT"], L_["HP"], L_["SLOTS"]
    assert G <= L_["G_max"] and G > JT
    per = U // G
    pc = min(PC, per)
    hc = min(HC + S // 16, per - pc)
    P = min(HP, G)
    starts = [cta_start(c, U, G, P, pc, JT, hc) for c in range(G + 1)]
    assert starts[0] == 0 and starts[G] == U
    assert all(starts[c] <= starts[c + 1] for c in range(G))

    slot_owner = {}
    for c in range(G):
        a, b = starts[c], starts[c + 1]
        L = b - a
        if L == 0:
            continue
        ta = a // S
        ws = [warp_start(a, L, w) for w in range(WARPS + 1)]
        assert ws[0] == a and ws[WARPS] == b
        assert all(ws[w] <= ws[w + 1] for w in range(WARPS))
        for w in range(WARPS):
            aw, bw = ws[w], ws[w + 1]
            for u in range(aw, bw):
                assert warp_owner(a, L, u) == w
            if aw == bw:
                continue
            for t in range(aw // S, (bw - 1) // S + 1):
                slot = (t - ta) + w
                assert 0 <= slot < SLOTS, (c, w, t, slot, SLOTS)
                key = (c, slot)
                assert key not in slot_owner, (key, slot_owner[key], (w, t))
                slot_owner[key] = (w, t)
        for u in (a, (a + b) // 2, b - 1):
            assert cta_owner(starts, G, u) == c

    # the finisher of each tile and the CTAs its pieces come from
    for t in range(L_["T"]):
        first, last = t * S, (t + 1) * S - 1
        c_first, c_last = cta_owner(starts, G, first), cta_owner(starts, G, last)
        assert c_first <= c_last
        assert starts[c_first] <= first < starts[c_first + 1]
        assert starts[c_last] <= last < starts[c_last + 1]
        for c in range(c_first + 1, c_last):   # CTAs in between lie inside the tile (or hold nothing)
            assert starts[c] >= first and starts[c + 1] <= last + 1


def test_slots_cover_the_longest_range():
    """The slot count is sized at one CTA per SM; more CTAs only shorten the
    ranges, so the two-CTA launch never needs more slots than the layout holds."""
    for N, K, r in itertools.product([4096, 11008, 22016], [4096, 11008, 22016], [16, 64]):
        L_ = layout(N, K, r)
        S, U, JT, HP = L_["S"], L_["U"], L_["JT"], L_["HP"]
        for G in (SMS, 2 * SMS):
            per = U // G
            pc = min(PC, per)
            hc = min(HC + S // 16, per - pc)
            starts = [cta_start(c, U, G, min(HP, G), pc, JT, hc) for c in range(G + 1)]
            longest = max(starts[c + 1] - starts[c] for c in range(G))
            assert ceil_div(longest, S) + 1 + (WARPS - 1) <= L_["SLOTS"]
