"""Exact-rational pins of the oracle's rounding chain (CPU only).

"QLoRA: fine-tuning a 65B model on one GPU", section "NormalFloat, double
quantization, paged optimizers": every weight is divided by its block's
absmax, mapped to the nearest of 16 levels, and the block constants are kept in
8 bits under a coarser constant; section "Where the memory goes": each pass
expands the stored weight back to 16 bits.  The readings fix each step's
rounding (every step one IEEE fp32 round-to-nearest-even, the 16-bit type bf16):

    normalize                 n   = fl32(w / a_b)                (0 when a_b = 0)
    dequantize_absmax         a'  = fl32(q_b * S_g)
    dequantize_absmax_signed  a'  = fl32(fl32(q_b * S_g) + mu)
    dequantize_nf4_bits       W'  = bf16(fl32(v_code * a'_b))

Each test recomputes the step from the exact rational value of its operands
(Python ``Fraction``), rounds with tests/exact.py's own rounding routines, and
compares bit patterns, on at least 10^5 elements over several groups
(partial groups, sub-normal constants, signed zeros included).  Each test
also feeds its check a copy of the oracle step with one rounding slip
planted (reciprocal-multiply, a fused multiply-add, one rounding where the
reading has two, a wrong group index) and requires that the check rejects it,
so a pin that could not see such a slip would fail here.
"""

from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4
from tests.exact import bf16_bits_exact, f32_rne, nearest_level_exact

F32_TINY = np.float32(1e-40)          # sub-normal


def _f32_bits(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)


def _bits(x) -> int:
    """fp32 bit pattern of one value."""
    return int(np.array(x, dtype=np.float32).view(np.uint32))


def _fr(x) -> Fraction:
    return Fraction(float(x))


# --------------------------------------------------------------------------- normalize

def _normalize_inputs(n_elems=100_000, seed=41):
    rng = np.random.default_rng(seed)
    w = rng.standard_normal(n_elems).astype(np.float32) * np.float32(0.02)
    w[5::97] = -0.0
    w[7::101] = 0.0
    w[11::89] *= np.float32(1e-36)                      # sub-normal weights
    w[64 * 3: 64 * 4] = 0.0                             # an all-zero block (a_b = 0)
    w[64 * 5: 64 * 6] = -0.0                            # all negative zeros
    w[64 * 7: 64 * 8] *= np.float32(1e-37)              # a block of sub-normal magnitude
    return w


def _check_normalize(fn, w) -> int:
    a = nf4.block_absmax(w)
    n = np.asarray(fn(w, a), dtype=np.float32)
    bad = 0
    for i in range(w.size):
        ab = a[i // 64]
        if ab == 0:
            exp = np.float32(0.0)
        elif w[i] == 0:
            exp = np.float32(-0.0) if np.signbit(w[i]) else np.float32(0.0)
        else:
            exp = np.float32(f32_rne(_fr(w[i]) / _fr(ab)))
        bad += int(_bits(exp) != _bits(n[i]))
    return bad


def _normalize_reciprocal(w_flat, absmax):
    """Planted slip: multiply by fl32(1 / a_b) instead of dividing."""
    w = np.asarray(w_flat, np.float32)
    a = np.repeat(absmax, 64)[: w.size]
    out = np.zeros_like(w)
    nz = a != 0
    out[nz] = w[nz] * (np.float32(1.0) / a[nz])
    return out


def test_normalize_exact():
    w = _normalize_inputs()
    assert _check_normalize(nf4.normalize, w) == 0


def test_normalize_pin_sees_reciprocal_multiply():
    w = _normalize_inputs(20_000, seed=42)
    assert _check_normalize(_normalize_reciprocal, w) > 0


# --------------------------------------------------------------------------- plain block constants

def _plain_constant_inputs(n_blocks=100_000 + 77, seed=43):
    """q in 0..255 with S per group of 256 blocks: ordinary, sub-normal and zero
    scales, and q extremes; the last group is partial."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 256, n_blocks).astype(np.uint8)
    q[::53] = 255
    q[1::59] = 0
    ng = -(-n_blocks // 256)
    S = (np.abs(rng.standard_normal(ng)).astype(np.float32) * np.float32(3e-4)).astype(np.float32)
    S[3] = F32_TINY
    S[5] = np.float32(2.0 ** -140)
    S[7] = 0.0
    S[9] = np.float32(np.finfo(np.float32).tiny)        # smallest normal
    return q, S


def _check_plain_constants(fn, q, S) -> int:
    got = _f32_bits(fn(q, S))
    bad = 0
    for b in range(q.size):
        exp = np.float32(f32_rne(Fraction(int(q[b])) * _fr(S[b // 256])))
        bad += int(_bits(exp) != int(got[b]))
    return bad


def _plain_constants_wrong_group(q, S):
    """Planted slip: group index from 255 blocks instead of 256."""
    Sb = np.asarray(S, np.float32)[np.minimum(np.arange(q.size) // 255, S.size - 1)]
    return (q.astype(np.float32) * Sb).astype(np.float32)


def _plain_constants_truncated(q, S):
    """Planted slip: the product truncated toward zero instead of rounded."""
    Sb = np.repeat(np.asarray(S, np.float32), 256)[: q.size].astype(np.float64)
    exact = q.astype(np.float64) * Sb                    # exact: 8 x 24 bits
    r = exact.astype(np.float32)
    over = np.abs(r.astype(np.float64)) > np.abs(exact)
    r[over] = np.nextafter(r[over], np.float32(0))
    return r


def test_dequantize_absmax_exact():
    q, S = _plain_constant_inputs()
    assert _check_plain_constants(nf4.dequantize_absmax, q, S) == 0


def test_dequantize_absmax_pin_sees_slips():
    q, S = _plain_constant_inputs(5000, seed=44)
    assert _check_plain_constants(_plain_constants_wrong_group, q, S) > 0
    assert _check_plain_constants(_plain_constants_truncated, q, S) > 0


# --------------------------------------------------------------------------- signed block constants

def _signed_constant_inputs(n_blocks=100_000 + 33, seed=45):
    """int8 codes -127..127 (and the never-written -128 bit pattern), scales and
    a mean of the same magnitude as q S, so the sum rounds in most elements."""
    rng = np.random.default_rng(seed)
    qi = rng.integers(-127, 128, n_blocks).astype(np.int8)
    qi[::61] = 127
    qi[1::67] = -127
    qi[2::71] = 0
    ng = -(-n_blocks // 256)
    S = (np.abs(rng.standard_normal(ng)).astype(np.float32) * np.float32(1e-4)).astype(np.float32)
    S[4] = F32_TINY
    S[6] = 0.0
    mus = [np.float32(0.0123), np.float32(0.0), np.float32(-3.7e-3), F32_TINY]
    return qi.view(np.uint8), S, mus


def _check_signed_constants(fn, q, S, mu) -> int:
    got = _f32_bits(fn(q, S, mu))
    qi = q.view(np.int8)
    bad = 0
    for b in range(q.size):
        p = f32_rne(Fraction(int(qi[b])) * _fr(S[b // 256]))        # fl32(q S)
        # sign of an exact zero sum: (+0) + (-0) = +0, (-0) + (-0) = -0 in round-to-nearest
        pz = np.signbit(np.float32(p)) if p == 0 else False
        total = Fraction(p) + _fr(mu)
        if total == 0:
            neg = bool(pz and np.signbit(mu)) if (p == 0 and mu == 0) else False
            exp = np.float32(-0.0) if neg else np.float32(0.0)
        else:
            exp = np.float32(f32_rne(total))
        bad += int(_bits(exp) != int(got[b]))
    return bad


def _signed_constants_fused(q, S, mu):
    """Planted slip: q S + mu with one rounding (a fused multiply-add)."""
    qi = np.asarray(q, np.uint8).view(np.int8).astype(np.float64)
    Sb = np.repeat(np.asarray(S, np.float32), 256)[: qi.size].astype(np.float64)
    # q S is exact in fp64 (8 x 24 bits); adding mu in fp64 then rounding to fp32 is a
    # double rounding that equals one correct rounding except in rare tie cases
    return (qi * Sb + np.float64(mu)).astype(np.float32)


def test_dequantize_absmax_signed_exact():
    q, S, mus = _signed_constant_inputs()
    assert _check_signed_constants(nf4.dequantize_absmax_signed, q, S, mus[0]) == 0
    for mu in mus[1:]:   # the other means on a fifth of the blocks
        assert _check_signed_constants(nf4.dequantize_absmax_signed, q[:20_000], S, mu) == 0, mu


def test_dequantize_absmax_signed_pin_sees_fused_rounding():
    q, S, mus = _signed_constant_inputs(20_000, seed=46)
    assert _check_signed_constants(_signed_constants_fused, q, S, mus[0]) > 0


# --------------------------------------------------------------------------- dequantized weight

def _tie_constructed_blocks(levels, count, seed):
    """(code, a') pairs whose fp32 product lands exactly on a bf16 rounding tie
    (low 16 bits 0x8000) while the exact product does not: one rounding of the
    exact product and the reading's two roundings (fp32, then bf16) disagree on
    about half of them."""
    rng = np.random.default_rng(seed)
    out = []
    nz = [c for c in range(16) if levels[c] != 0]
    while len(out) < count:
        c = int(rng.choice(nz))
        v = levels[c]
        target_bits = (int(rng.integers(0x3C00, 0x3E00)) << 16) | 0x8000      # |t| ~ 2^-7 .. 2^-3
        t = np.uint32(target_bits).view(np.float32)
        a = np.float32(np.float64(t) / np.float64(v))
        a = np.float32(abs(a))
        if a == 0 or not np.isfinite(a):
            continue
        prod = np.float32(v) * a
        exact = _fr(v) * _fr(a)
        if _bits(prod) & 0xFFFF == 0x8000 and Fraction(float(prod)) != exact:
            out.append((c, a))
    return out


def _dequant_inputs(fmt, dq, n=100_000 + 64 * 3 + 5, seed=47):
    """Random codes, 8-bit constants and group scales over several groups (the
    last partial, odd element count), sub-normal and zero scales, and the
    constructed tie cases placed as whole blocks with q = 1 (a' = S)."""
    rng = np.random.default_rng(seed)
    levels = nf4.codebook(fmt)
    codes = rng.integers(0, 16, n).astype(np.uint8)
    nb = -(-n // 64)
    ng = -(-nb // 256)
    q = rng.integers(0, 256, nb).astype(np.uint8)
    if dq == "signed":
        q = rng.integers(-127, 128, nb).astype(np.int8).view(np.uint8)
    S = (np.abs(rng.standard_normal(ng)).astype(np.float32) * np.float32(2e-4)).astype(np.float32)
    S[1] = F32_TINY
    S[2] = 0.0
    mu = np.float32(0.0117) if dq == "signed" else np.float32(0.0)
    if dq == "plain":
        # group 3 holds the tie cases: one block per constructed pair, q = 1, S = a'
        # would need one S per block, so use one group per pair for the first few
        ties = _tie_constructed_blocks(levels, min(ng - 4, 40), seed + 1)
        for i, (c, a) in enumerate(ties):
            g = 4 + i
            S[g] = a
            blk = g * 256
            if blk * 64 + 64 > n:
                break
            q[blk] = 1
            codes[blk * 64: blk * 64 + 64] = c
    return codes, q, S, mu, levels


def _check_dequant(fn, fmt, dq, codes, q, S, mu, levels, elems=None) -> int:
    n = codes.size
    packed = nf4.pack_nibbles(codes)
    got = np.asarray(fn(packed, q, S, (n,), fmt, dq, mu), dtype=np.uint16).ravel()
    qi = q.view(np.int8) if dq == "signed" else q
    bad = 0
    cache = {}
    for e in (range(n) if elems is None else elems):
        b = e // 64
        if b not in cache:
            p = f32_rne(Fraction(int(qi[b])) * _fr(S[b // 256]))
            if dq == "signed":
                tot = Fraction(p) + _fr(mu)
                a = np.float32(f32_rne(tot)) if tot != 0 else np.float32(0.0)
            else:
                a = np.float32(p)
            cache = {b: a}
        a = cache[b]
        v = levels[codes[e]]
        t = f32_rne(_fr(v) * _fr(a))                  # fl32(v a'), exact rational
        neg_zero = t == 0 and (bool(np.signbit(v)) != bool(np.signbit(a)))
        exp = bf16_bits_exact(Fraction(t), negative_zero=neg_zero)
        bad += int(exp != int(got[e]))
    return bad


def _dequant_single_rounding(codes, absmax_q, group_scale, shape, fmt="nf4", dq="plain", offset=0.0):
    """Planted slip: v a' formed exactly (in fp64, 24 x 24 bits) and rounded
    once, straight to 8 significant bits (normal range)."""
    numel = int(np.prod(shape))
    c = nf4.unpack_nibbles(codes, numel)
    v = nf4.codebook(fmt)[c].astype(np.float64)
    a = (nf4.dequantize_absmax(absmax_q, group_scale) if dq == "plain"
         else nf4.dequantize_absmax_signed(absmax_q, group_scale, offset))
    p = v * np.repeat(a, 64)[:numel].astype(np.float64)
    m, e = np.frexp(p)
    r = np.ldexp(np.rint(m * 256.0) / 256.0, e).astype(np.float32)   # 8 bits: exact in fp32
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def _dequant_high_nibble_first(codes, absmax_q, group_scale, shape, fmt="nf4", dq="plain", offset=0.0):
    """Planted slip: the two codes of a byte swapped."""
    p = np.asarray(codes, np.uint8)
    swapped = ((p >> 4) | (p << 4)).astype(np.uint8)
    return nf4.dequantize_nf4_bits(swapped, absmax_q, group_scale, shape, fmt, dq, offset)


@pytest.mark.parametrize("fmt,dq", [("nf4", "plain"), ("nf4", "signed"), ("fp4", "plain"), ("int4", "plain")])
def test_dequantize_nf4_bits_exact(fmt, dq):
    n = 100_000 + 64 * 3 + 5 if (fmt, dq) == ("nf4", "plain") else 64 * 256 * 3 + 64 * 5 + 7
    codes, q, S, mu, levels = _dequant_inputs(fmt, dq, n=n)
    assert _check_dequant(nf4.dequantize_nf4_bits, fmt, dq, codes, q, S, mu, levels) == 0


def test_dequantize_pin_sees_single_rounding_and_nibble_order():
    codes, q, S, mu, levels = _dequant_inputs("nf4", "plain", n=64 * 256 * 12 + 64, seed=48)
    # the constructed ties (first block of groups 4..) are where one rounding and two roundings part
    ties = [e for g in range(4, S.size) for e in range(g * 256 * 64, g * 256 * 64 + 64) if e < codes.size]
    assert _check_dequant(_dequant_single_rounding, "nf4", "plain", codes, q, S, mu, levels, ties) > 0
    assert _check_dequant(_dequant_high_nibble_first, "nf4", "plain", codes, q, S, mu, levels, range(4000)) > 0


def test_tie_cases_are_real():
    """The constructed cases do sit on a bf16 tie after the fp32 rounding, and
    one rounding of the exact product goes the other way for some of them."""
    lv = nf4.codebook("nf4")
    ties = _tie_constructed_blocks(lv, 60, seed=49)
    differ = 0
    for c, a in ties:
        t = f32_rne(_fr(lv[c]) * _fr(a))
        assert _bits(t) & 0xFFFF == 0x8000
        differ += int(bf16_bits_exact(Fraction(t)) != bf16_bits_exact(_fr(lv[c]) * _fr(a)))
    assert differ >= 10


# --------------------------------------------------------------------------- encode from raw weights

def _encode_exact(w, levels):
    """w -> a_b -> n -> code, every step on exact rationals: a_b = max |w| of
    the block, n = fl32(w / a_b) by an exact rounding, code = the nearest level
    with ties to the lower index by exact distances."""
    w = np.asarray(w, np.float32)
    codes = []
    for b0 in range(0, w.size, 64):
        blk = w[b0:b0 + 64]
        a = max((abs(_fr(x)) for x in blk), default=Fraction(0))
        for x in blk:
            n = 0.0 if a == 0 else f32_rne(_fr(x) / a)
            codes.append(nearest_level_exact(np.float32(n), levels))
    return np.array(codes, np.uint8)


def _adversarial_blocks(levels, rng, nblocks):
    """Blocks whose absmax is a power of two or a random value and whose other
    weights are placed at each midpoint of two levels times a_b, and one ulp
    either side, so n lands on, just below and just above every threshold."""
    out = []
    for i in range(nblocks):
        a = np.float32(2.0 ** int(rng.integers(-8, 0))) if i % 2 == 0 else \
            np.float32(abs(rng.standard_normal()) * 0.05 + 1e-3)
        blk = [a if i % 3 else -a]
        for j in range(15):
            mid = (_fr(levels[j]) + _fr(levels[j + 1])) / 2
            m = np.float32(f32_rne(mid * _fr(a)))
            blk += [m, np.nextafter(m, np.float32(-1)), np.nextafter(m, np.float32(1))]
        blk += list(rng.uniform(-1, 1, 64 - len(blk)).astype(np.float32) * a)
        out.append(np.array(blk[:64], np.float32))
    return np.concatenate(out)


@pytest.mark.parametrize("fmt", nf4.FORMATS)
def test_encode_from_raw_weights_bruteforce(fmt):
    rng = np.random.default_rng(50)
    lv = nf4.codebook(fmt)
    w = np.concatenate([
        _adversarial_blocks(lv, rng, 24),
        rng.standard_normal(64 * 8 + 21).astype(np.float32) * np.float32(0.02),   # ends in a partial block
    ])
    w[64 * 30 + 3] = -0.0
    got = nf4.unpack_nibbles(nf4.quantize_nf4(w, fmt)["codes"], w.size)
    assert np.array_equal(got, _encode_exact(w, lv))


# --------------------------------------------------------------------------- equal share (reported)

def test_equal_share_report(capsys):
    """The pages: the NF4 levels sit at normal quantiles, so Gaussian weights use
    every level about equally.  Absmax scaling makes it approximate (the block
    maximum always takes an end level), so this is a report with loose bounds,
    not a parity gate: the code entropy and the largest / smallest level share
    on a Gaussian 1024 x 1024 weight, for the three tables."""
    rng = np.random.default_rng(51)
    W = rng.standard_normal((1024, 1024)).astype(np.float32) * np.float32(0.02)
    rep = {}
    for fmt in nf4.FORMATS:
        c = nf4.unpack_nibbles(nf4.quantize_nf4(W, fmt)["codes"], W.size)
        h = np.bincount(c, minlength=16).astype(np.float64) / c.size
        used = h[h > 0]
        rep[fmt] = (float(-(used * np.log2(used)).sum()), float(used.max() / used.min()))
    with capsys.disabled():
        print("\ncode entropy (bits) / max:min level share on Gaussian weights: "
              + ", ".join(f"{k} {e:.3f} / {r:.2f}" for k, (e, r) in rep.items()))
    assert rep["nf4"][0] > rep["fp4"][0] and rep["nf4"][0] > rep["int4"][0]
    assert rep["nf4"][0] > 3.7
