"""Pins for the NF4 / double-quantization oracle (CPU only).

Each test checks the oracle against something other than itself: closed forms,
exact rational brute force, library routines for special cases, invariants the
pages fix, or the pages' own figures (tests/golden/page_figures.json).
"""

import json
import os
import statistics
from fractions import Fraction

import numpy as np
import pytest
import scipy.special as sps
import torch

from oracle import nf4
from tests.exact import f32_rne, nearest_level_exact, round_half_even

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- codebook

def _levels_from_quantile(qfun):
    """Rebuild the 16 levels with another quantile routine (float64)."""
    d = 1.0 - (1.0 / 32 + 1.0 / 30) / 2
    pos = [qfun(d + (0.5 - d) * i / 8) for i in range(8)]
    neg = [-qfun(d + (0.5 - d) * i / 7) for i in range(7)]
    vals = np.array(sorted(pos + neg + [0.0]), dtype=np.float64)
    return (vals / np.max(np.abs(vals))).astype(np.float32)


def test_codebook_invariants():
    v = nf4.nf4_codebook()
    assert v.dtype == np.float32 and v.size == 16
    assert np.all(np.diff(v) > 0), "levels strictly increasing"
    assert v[0] == np.float32(-1.0) and v[15] == np.float32(1.0)
    assert v[7] == 0.0 and not np.signbit(v[7]), "exact +0 level"
    assert np.sum(v < 0) == 7 and np.sum(v > 0) == 8


def test_codebook_quantile_routines_agree_bitwise():
    v = nf4.nf4_codebook().view(np.uint32)
    nd = statistics.NormalDist()
    assert np.array_equal(_levels_from_quantile(nd.inv_cdf).view(np.uint32), v)
    assert np.array_equal(_levels_from_quantile(sps.ndtri).view(np.uint32), v)


def test_codebook_equal_mass_by_forward_cdf():
    """Closed form of the construction checked with the forward CDF (a different
    routine than the quantile): on each side the levels, scaled back by the
    outer quantile, cut the normal into equal probability slices."""
    v = nf4.nf4_codebook().astype(np.float64)
    d = 1.0 - (1.0 / 32 + 1.0 / 30) / 2
    top = sps.ndtri(d)
    pos = np.sort(v[v > 0])[::-1]                 # 1 .. smallest positive
    cdf_pos = sps.ndtr(pos * top)
    expect_pos = d + (0.5 - d) * np.arange(8) / 8
    assert np.allclose(cdf_pos, expect_pos, atol=2e-7)
    neg = np.sort(-v[v < 0])[::-1]
    cdf_neg = sps.ndtr(neg * top)
    expect_neg = d + (0.5 - d) * np.arange(7) / 7
    assert np.allclose(cdf_neg, expect_neg, atol=2e-7)


def test_codebook_robust_to_quantile_error():
    """Every level is far (in fp32 ulps) from an fp32 rounding boundary, so the
    fp32 table does not depend on the last digits of the quantile routine."""
    for lv in nf4.nf4_levels_exact():
        x = float(lv)
        f = np.float32(x)
        if f == 0:
            continue
        ulp = float(np.spacing(np.float32(abs(f))))
        frac = abs(x - float(f)) / ulp
        assert frac < 0.49, frac


def test_codebook_golden():
    with open(os.path.join(GOLDEN, "nf4_codebook_f32.txt")) as fh:
        bits = [int(line.split()[0], 16) for line in fh if line.strip() and not line.startswith("#")]
    assert nf4.nf4_codebook().view(np.uint32).tolist() == bits


# --------------------------------------------------------------------------- bf16

def test_bf16_rne_matches_torch():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(3e-2),
        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-39),   # subnormals
        # exact ties at bf16 precision, both parities of the kept part
        (np.arange(0x3F800000, 0x3F800000 + 4096, dtype=np.uint32) * 0 + 0x3F808000
         + (np.arange(4096, dtype=np.uint32) << 16)).view(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0], np.float32),
    ])
    ours = nf4.bf16_rne_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------- nearest code

def test_nearest_code_bruteforce_random_and_midpoints():
    v = nf4.nf4_codebook()
    rng = np.random.default_rng(11)
    pts = [rng.uniform(-1, 1, 3000).astype(np.float32)]
    for i in range(15):
        mid = (Fraction(float(v[i])) + Fraction(float(v[i + 1]))) / 2
        m32 = np.float32(float(mid))
        near = [m32]
        lo = hi = m32
        for _ in range(4):
            lo = np.nextafter(lo, np.float32(-2))
            hi = np.nextafter(hi, np.float32(2))
            near += [lo, hi]
        pts.append(np.array(near, np.float32))
    pts.append(v.copy())
    pts.append(np.array([0.0, -0.0, 1.0, -1.0, 1e-40, -1e-40], np.float32))
    n = np.concatenate(pts)
    got = nf4.nearest_code(n, v)
    exp = np.array([nearest_level_exact(x, v) for x in n], np.uint8)
    assert np.array_equal(got, exp)


def test_nearest_code_exact_tie_goes_low():
    """Construct levels whose midpoint is an exact fp32 value: the tie must pick
    the lower index."""
    lv = np.array([-1, -0.5, 0, 0.25, 0.5, 1] + [2 + i for i in range(10)], np.float32)
    got = nf4.nearest_code(np.array([0.125, 0.375, -0.25, -0.75], np.float32), lv)
    assert got.tolist() == [2, 3, 1, 0]


# --------------------------------------------------------------------------- packing

def test_pack_order_low_nibble_first():
    assert nf4.pack_nibbles(np.array([1, 2, 3], np.uint8)).tolist() == [0x21, 0x03]
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(nf4.unpack_nibbles(nf4.pack_nibbles(codes), 16), codes)


# --------------------------------------------------------------------------- absmax / encode

def test_block_absmax_partial_block():
    rng = np.random.default_rng(3)
    w = rng.standard_normal(64 * 3 + 10).astype(np.float32)
    a = nf4.block_absmax(w)
    assert a.size == 4
    for b in range(4):
        assert a[b] == np.max(np.abs(w[64 * b: 64 * b + 64]))


def test_quantize_special_cases():
    w = np.zeros(64 * 4, np.float32)
    w[0:64] = np.linspace(-0.3, 0.2, 64, dtype=np.float32)     # -absmax at element 0
    w[64:128] = np.linspace(-0.1, 0.7, 64, dtype=np.float32)   # +absmax at element 127
    # block 2 stays all zero (including a negative zero)
    w[130] = -0.0
    w[192:256] = 1e-3
    q = nf4.quantize_nf4(w)
    c = nf4.unpack_nibbles(q["codes"], w.size)
    assert c[0] == 0 and c[127] == 15
    assert np.all(c[128:192] == 7)
    assert np.all(c[192:256] == 15)


def test_roundtrip_exact_on_codebook_grid():
    """Weights on the NF4 grid times a = 255 * 2^j: S_g = 2^j exactly, q = 255,
    a' = a, so dequant(quant(W)) must equal bf16(W) bit for bit and the codes must
    reproduce the grid indices -- end to end through block, group and packing
    indexing (a wrong nibble order, block or group index breaks it)."""
    v = nf4.nf4_codebook()
    rng = np.random.default_rng(5)
    n_blocks = 256 * 2 + 24                       # 2 full groups + a partial one
    idx = rng.integers(0, 16, size=n_blocks * 64).astype(np.uint8)
    idx[::64] = 15                                # every block hits the top level
    scale = np.float32(255.0 * 2.0 ** -9)
    w = (v[idx] * scale).astype(np.float32).reshape(-1, 64 * 8)
    q = nf4.quantize_nf4(w)
    assert np.all(q["absmax_q"] == 255)
    assert np.all(q["group_scale"] == np.float32(2.0 ** -9))
    assert np.array_equal(nf4.unpack_nibbles(q["codes"], idx.size), idx)
    deq = nf4.dequantize_nf4(q)
    assert np.array_equal(deq, nf4.bf16_rne_bits(w))


def test_nonfinite_rejected():
    w = np.zeros(128, np.float32)
    w[5] = np.inf
    with pytest.raises(ValueError):
        nf4.quantize_nf4(w)
    w[5] = np.nan
    with pytest.raises(ValueError):
        nf4.quantize_nf4(w)


# --------------------------------------------------------------------------- double quantization

def _dq_bruteforce(a32):
    a = [Fraction(float(x)) for x in a32]
    out_q, out_S = [], []
    for g in range(0, len(a), 256):
        grp = a[g:g + 256]
        c = max(grp)
        S = f32_rne(c / 255)
        out_S.append(S)
        for x in grp:
            if S == 0:
                out_q.append(0)
            else:
                out_q.append(min(255, round_half_even(Fraction(f32_rne(x / Fraction(S))))))
    return np.array(out_q, np.uint8), np.array(out_S, np.float32)


def test_double_quant_bruteforce():
    rng = np.random.default_rng(9)
    a = np.abs(rng.standard_normal(256 * 3 + 40).astype(np.float32)) * np.float32(0.05)
    a[300] = 0.0
    a[256 * 3:] *= np.float32(1e-38)             # a tiny (subnormal-scale) last group
    q, S = nf4.double_quantize(a)
    qb, Sb = _dq_bruteforce(a)
    assert np.array_equal(S.view(np.uint32), Sb.view(np.uint32))
    assert np.array_equal(q, qb)


def test_double_quant_invariants():
    rng = np.random.default_rng(10)
    a = np.abs(rng.standard_normal(256 * 8).astype(np.float32)) * np.float32(0.04)
    q, S = nf4.double_quantize(a)
    ap = nf4.dequantize_absmax(q, S)
    for g in range(8):
        grp = a[256 * g: 256 * g + 256]
        assert q[256 * g + int(np.argmax(grp))] == 255
        err = np.abs(ap[256 * g: 256 * g + 256].astype(np.float64) - grp.astype(np.float64))
        assert np.all(err <= S[g] * 0.5 * (1 + 2e-6) + 4 * np.spacing(grp.astype(np.float32)))
    const = np.full(256, np.float32(0.0123))
    qc, _ = nf4.double_quantize(const)
    assert np.all(qc == 255)
    qz, Sz = nf4.double_quantize(np.zeros(256, np.float32))
    assert np.all(qz == 0) and Sz[0] == 0


# --------------------------------------------------------------------------- dequant bound, footprint

def test_roundtrip_error_bound_gaussian():
    rng = np.random.default_rng(12)
    W = rng.standard_normal((64, 1024)).astype(np.float32) * np.float32(0.02)
    q = nf4.quantize_nf4(W)
    Wd = nf4.bf16_bits_to_f32(nf4.dequantize_nf4(q)).astype(np.float64).ravel()
    a = np.repeat(nf4.block_absmax(W), 64).astype(np.float64)
    ap = np.repeat(nf4.dequantize_absmax(q["absmax_q"], q["group_scale"]), 64).astype(np.float64)
    gap = np.max(np.diff(nf4.nf4_codebook().astype(np.float64))) / 2
    bound = gap * a * (1 + 1e-6) + np.abs(a - ap) + 2.0 ** -8 * np.abs(Wd) + 1e-30
    assert np.all(np.abs(W.ravel().astype(np.float64) - Wd) <= bound)
    assert gap < 0.152


def test_footprint_and_page_figures():
    """Footprint formula vs the pages' figures (tests/golden/page_figures.json)."""
    with open(os.path.join(GOLDEN, "page_figures.json")) as fh:
        fig = json.load(fh)
    n = 4096 * 4096
    assert nf4.footprint_bytes(n) == n // 2 + n // 64 + 4 * (n // 16384)
    bits = 8 * nf4.footprint_bytes(n) / n
    assert abs(bits - 4.127) < 1e-3
    # 16-bit storage of a 65B model is 130 GB (2 bytes per parameter).
    p65 = fig["params_65b"]
    assert p65 * 2 / 1e9 == fig["bf16_bytes_65b_gb"]
    # about four times smaller than 16-bit weights, within the rounding the page uses.
    ratio = 16 / bits
    assert abs(ratio - fig["compression_vs_16bit"]) < 0.5
    # 65B frozen base in NF4+DQ fits a single 48 GB GPU with room for adapters.
    assert p65 * bits / 8 / 1e9 < fig["single_gpu_gb"]


def test_partial_groups_layout_sizes():
    numel = 64 * 256 * 2 + 64 * 5 + 3
    w = np.random.default_rng(1).standard_normal(numel).astype(np.float32)
    q = nf4.quantize_nf4(w)
    assert q["codes"].size == (numel + 1) // 2
    assert q["absmax_q"].size == nf4.num_blocks(numel) == 256 * 2 + 6
    assert q["group_scale"].size == 3
    assert (q["codes"][-1] >> 4) == 0          # unused high nibble is zero


def test_golden_small_quantization():
    """Regression pin: the 256x256 seed-0 weight's quantization (written by
    tests/golden/make_golden.py from the oracle) must not drift."""
    import qlora_inputs as qi
    with open(os.path.join(GOLDEN, "small_quant_digest.json")) as fh:
        g = json.load(fh)
    W = qi.make_linear(qi.SMALL)["W"].numpy()
    q = nf4.quantize_nf4(W)
    import hashlib
    assert hashlib.sha256(q["codes"].tobytes()).hexdigest() == g["codes_sha256"]
    assert q["absmax_q"].tolist() == g["absmax_q"]
    assert [float(x).hex() for x in q["group_scale"]] == g["group_scale_hex"]
