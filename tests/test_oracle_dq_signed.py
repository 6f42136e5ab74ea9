"""Pins of the oracle's second double-quantization reading: the block
constants minus their tensor-wide mean, in signed 8-bit codes.

"QLoRA: fine-tuning a 65B model on one GPU", section "NormalFloat, double
quantization, paged optimizers" (the block constants are stored in 8 bits
under a coarser set of constants) leaves the 8-bit format open; this variant
centres the constants on their mean first.  The mean must not depend on a
summation order, so it is defined from the exact sum; these tests check the
oracle's integer route to that sum against exact rationals, against
math.fsum (Shewchuk's correctly rounded summation), against closed forms and
against cases where an ordinary floating-point sum would be wrong."""

import math
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4
from tests.exact import f32_rne, round_half_even


def _mean_bruteforce(a32):
    total = sum(Fraction(float(x)) for x in a32)
    s64 = float(total)                         # int / int true division: correctly rounded
    return np.float32(f32_rne(Fraction(s64 / float(len(a32)))))


def _awkward_constants(rng, n):
    """Non-negative fp32 values over the whole range: zeros, subnormals,
    normals from 2^-126 to 2^126 and a bulk of typical block constants."""
    a = np.abs(rng.standard_normal(n).astype(np.float32)) * np.float32(0.05)
    a[::17] = 0.0
    a[3::29] = np.float32(1e-44)                                   # subnormal
    a[5::31] = np.ldexp(np.float32(1.0), rng.integers(-126, 127, a[5::31].size)).astype(np.float32)
    a[7::37] = np.float32(np.finfo(np.float32).max)
    return a


def test_exact_sum_matches_rationals():
    rng = np.random.default_rng(31)
    a = _awkward_constants(rng, 3000)
    units = nf4.exact_sum_units(a)
    assert Fraction(units, 2 ** 149) == sum(Fraction(float(x)) for x in a)


def test_exact_sum_rounds_like_fsum():
    rng = np.random.default_rng(32)
    for n in (1, 7, 1000, 20000):
        a = _awkward_constants(rng, n)
        s64 = math.ldexp(float(nf4.exact_sum_units(a)), -149)
        assert s64 == math.fsum(a.astype(np.float64).tolist())


def test_mean_matches_bruteforce():
    rng = np.random.default_rng(33)
    for n in (1, 2, 255, 256, 257, 4099):
        a = _awkward_constants(rng, n)
        assert nf4.block_constant_mean(a).view(np.uint32) == _mean_bruteforce(a).view(np.uint32)
        b = np.abs(rng.standard_normal(n).astype(np.float32)) * np.float32(0.03)
        assert nf4.block_constant_mean(b).view(np.uint32) == _mean_bruteforce(b).view(np.uint32)


def test_mean_where_a_float_sum_is_wrong():
    # 2^60 then a thousand ones: an fp64 running sum drops every one (2^60 + 1 == 2^60),
    # the exact sum keeps them and rounds once: 2^60 + 1000 -> 2^60 + 1024 in fp64.
    a = np.array([2.0 ** 60] + [1.0] * 1000, np.float32)
    run = 0.0
    for x in a.tolist():
        run += x
    assert run == 2.0 ** 60
    assert math.ldexp(float(nf4.exact_sum_units(a)), -149) == 2.0 ** 60 + 1024
    assert nf4.block_constant_mean(a) == np.float32((2.0 ** 60 + 1024) / 1001)


def test_mean_closed_forms_and_order():
    v = np.float32(0.0371)
    for n in (1, 3, 256, 10001):
        assert nf4.block_constant_mean(np.full(n, v)) == v              # n v exact in fp64, / n exact
    assert nf4.block_constant_mean(np.zeros(5, np.float32)) == 0.0
    assert nf4.block_constant_mean(np.array([1.0, 2.0], np.float32)) == np.float32(1.5)
    rng = np.random.default_rng(34)
    a = _awkward_constants(rng, 5000)
    m = nf4.block_constant_mean(a)
    for _ in range(3):
        assert nf4.block_constant_mean(rng.permutation(a)).view(np.uint32) == m.view(np.uint32)
    with pytest.raises(ValueError):
        nf4.exact_sum_units(np.array([-1.0], np.float32))


def _dq_signed_bruteforce(a32):
    mu = _mean_bruteforce(a32)
    c = [f32_rne(Fraction(float(x)) - Fraction(float(mu))) for x in a32]
    out_q, out_S = [], []
    for g in range(0, len(c), 256):
        grp = c[g:g + 256]
        S = f32_rne(Fraction(max(abs(x) for x in grp)) / 127)
        out_S.append(S)
        for x in grp:
            if S == 0:
                out_q.append(0)
            else:
                r = round_half_even(Fraction(f32_rne(Fraction(x) / Fraction(S))))
                out_q.append(max(-127, min(127, r)))
    return np.array(out_q, np.int8).view(np.uint8), np.array(out_S, np.float32), mu


def test_signed_double_quant_bruteforce():
    rng = np.random.default_rng(35)
    a = np.abs(rng.standard_normal(256 * 3 + 40).astype(np.float32)) * np.float32(0.05)
    a[300] = 0.0
    a[600:610] = np.float32(0.2)                  # outliers: one group's scale is set by them
    a[256 * 3:] *= np.float32(1e-30)              # a tiny last group, far below the mean
    q, S, mu = nf4.double_quantize_signed(a)
    qb, Sb, mub = _dq_signed_bruteforce(a)
    assert mu.view(np.uint32) == mub.view(np.uint32)
    assert np.array_equal(S.view(np.uint32), Sb.view(np.uint32))
    assert np.array_equal(q, qb)


def test_signed_double_quant_invariants():
    rng = np.random.default_rng(36)
    a = np.abs(rng.standard_normal(256 * 8).astype(np.float32)) * np.float32(0.04)
    q, S, mu = nf4.double_quantize_signed(a)
    qi = q.view(np.int8)
    ap = nf4.dequantize_absmax_signed(q, S, mu)
    c = (a - mu).astype(np.float32)
    assert qi.min() >= -127
    for g in range(8):
        sl = slice(256 * g, 256 * g + 256)
        k = int(np.argmax(np.abs(c[sl])))
        assert abs(int(qi[sl][k])) == 127 and np.sign(qi[sl][k]) == np.sign(c[sl][k])
        err = np.abs(ap[sl].astype(np.float64) - a[sl].astype(np.float64))
        # half a step of S_g, plus the fp32 roundings of a - mu, q S and q S + mu
        assert np.all(err <= S[g] * 0.5 * (1 + 2e-6) + 4 * np.spacing(np.maximum(a[sl], mu)))
    # a group whose constants all equal the mean: no deviation to code
    flat = np.full(512, np.float32(0.02))
    qf, Sf, muf = nf4.double_quantize_signed(flat)
    assert muf == np.float32(0.02) and np.all(Sf == 0) and np.all(qf == 0)
    assert np.all(nf4.dequantize_absmax_signed(qf, Sf, muf) == np.float32(0.02))


def test_signed_variant_keeps_codes_and_shrinks_constant_error():
    rng = np.random.default_rng(37)
    W = rng.standard_normal((128, 2048)).astype(np.float32) * np.float32(0.02)
    qp = nf4.quantize_nf4(W)
    qs = nf4.quantize_nf4(W, dq="signed")
    assert np.array_equal(qp["codes"], qs["codes"])      # codes use the exact block absmax either way
    a = nf4.block_absmax(W.ravel()).astype(np.float64)
    ep = np.abs(nf4.dequantize_absmax(qp["absmax_q"], qp["group_scale"]) - a).mean()
    es = np.abs(nf4.dequantize_absmax_signed(qs["absmax_q"], qs["group_scale"], qs["offset"]) - a).mean()
    # Gaussian blocks: constants near 2.4 sigma with a spread well under their size, so the
    # signed step max|a - mu| / 127 is finer than max a / 255.
    assert es < 0.9 * ep
    # the weight error is dominated by the 4-bit codes: the two readings agree to 1 %
    rp = nf4.reconstruction_error(W)
    rs = nf4.reconstruction_error(W, dq="signed")
    assert abs(rs - rp) <= 0.01 * rp
    with pytest.raises(ValueError):
        nf4.quantize_nf4(W, dq="other")
