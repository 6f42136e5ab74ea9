"""The plain 4-bit float and integer tables (the types the pages compare NF4
against) in the oracle and in the library, pinned on the CPU:

- the FP4 levels equal the values of the 16 e2m1 bit patterns (decoded here
  from the sign / exponent / mantissa fields), scaled so the largest is 1;
- the Int4 levels are the 15 equally spaced values k/7 plus -8/7;
- the library's exported levels are bit-identical to the oracle's, and its
  threshold encoding agrees with the oracle's nearest-level encoding (ties to
  the lower index) on every fp32 value within 3 ulps of every threshold;
- on Gaussian weights NF4 reconstructs with less error than both (the pages'
  ablation statement, as a reconstruction-error proxy).
"""

import ctypes
from fractions import Fraction

import numpy as np
import pytest

from oracle import nf4

FMT_ID = {"nf4": 0, "fp4": 1, "int4": 2}


def e2m1_value(bits: int) -> Fraction:
    """Value of a 4-bit e2m1 pattern: sign bit 3, exponent bits 2..1 (bias 1),
    mantissa bit 0; exponent 0 is subnormal (0.m x 2^0)."""
    sign = -1 if bits & 8 else 1
    e = (bits >> 1) & 3
    m = bits & 1
    mag = Fraction(m, 2) if e == 0 else (1 + Fraction(m, 2)) * Fraction(2) ** (e - 1)
    return sign * mag


def test_fp4_levels_are_the_e2m1_values():
    vals = sorted({e2m1_value(b) for b in range(16)})
    assert len(vals) == 15 and max(vals) == 6 and min(vals) == -6       # +-0 coincide
    lv = nf4.codebook("fp4")
    got = [Fraction(float(x)) for x in lv]
    # every level is the fp32 rounding of an e2m1 value / 6, each value used, both zeros present
    want = [np.float32(float(v / 6)) for v in vals]
    assert sorted({float(x) for x in lv}) == sorted({float(w) for w in want})
    assert np.signbit(lv[7]) and not np.signbit(lv[8]) and lv[7] == 0 and lv[8] == 0
    assert all(a <= b for a, b in zip(got, got[1:]))
    assert lv[0] == -1 and lv[15] == 1


def test_int4_levels_are_an_even_grid():
    lv = nf4.codebook("int4").astype(np.float64)
    assert lv[8] == 0 and lv[1] == -1 and lv[15] == 1
    steps = np.diff(lv)
    assert np.allclose(steps, 1 / 7, rtol=0, atol=1e-7)
    for c in range(16):
        assert Fraction(float(lv[c])) == Fraction(float(np.float32(float(Fraction(c - 8, 7)))))


def test_fp4_encoding_never_emits_the_positive_zero():
    rng = np.random.default_rng(3)
    n = np.concatenate([rng.uniform(-1, 1, 20000).astype(np.float32),
                        np.array([0.0, -0.0, 1e-30, -1e-30, 1 / 24, -1 / 24], np.float32)])
    codes = nf4.nearest_code(n, nf4.codebook("fp4"))
    assert not np.any(codes == 8)
    assert np.all(codes[np.abs(n) < np.float32(1 / 24) * 0.999] == 7)


def test_reconstruction_error_nf4_beats_fp4_and_int4_on_gaussian_weights():
    rng = np.random.default_rng(11)
    W = rng.standard_normal((512, 1024), dtype=np.float32) * np.float32(0.02)
    err = {f: nf4.reconstruction_error(W, f) for f in nf4.FORMATS}
    assert err["nf4"] < err["fp4"] and err["nf4"] < err["int4"], err


def _lib_tables(lib, fmt):
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    assert lib.load().qlora_format_codebook(FMT_ID[fmt], lv, th) == 0
    return np.array(lv, np.float32), np.array(th, np.float32)


@pytest.mark.parametrize("fmt", nf4.FORMATS)
def test_library_tables_match_the_oracle(lib, fmt):
    lv, th = _lib_tables(lib, fmt)
    assert np.array_equal(lv.view(np.uint32), nf4.codebook(fmt).view(np.uint32))
    # threshold encoding == nearest level with ties low, on a dense set of values around every threshold
    probes = []
    for t in th:
        v = np.float32(t)
        for _ in range(3):
            v = np.nextafter(v, np.float32(-np.inf))
        for _ in range(7):   # t - 3 ulp .. t + 3 ulp
            probes.append(v)
            v = np.nextafter(v, np.float32(np.inf))
    probes += [np.float32(v) for v in (-1.0, -0.0, 0.0, 1.0)]
    n = np.array(probes, np.float32)
    by_threshold = (n[:, None] > th[None, :]).sum(axis=1)
    assert np.array_equal(by_threshold, nf4.nearest_code(n, nf4.codebook(fmt)).astype(np.int64))


def test_library_rejects_unknown_formats(lib):
    lv = (ctypes.c_float * 16)()
    assert lib.load().qlora_format_codebook(3, lv, None) == 1
    assert lib.load().qlora_format_codebook(-1, lv, None) == 1


@pytest.mark.parametrize("fmt", nf4.FORMATS)
def test_fast_encoder_equals_the_argmin_definition(fmt):
    """The midpoint-count encoder used for large weights returns the same code
    as the nearest-level argmin (ties low) on dense probes around every
    midpoint and on random values."""
    lv = nf4.codebook(fmt)
    probes = []
    for i in range(15):
        v = np.float32((np.float64(lv[i]) + np.float64(lv[i + 1])) / 2)
        for _ in range(4):
            v = np.nextafter(v, np.float32(-np.inf))
        for _ in range(9):
            probes.append(v)
            v = np.nextafter(v, np.float32(np.inf))
    rng = np.random.default_rng(5)
    n = np.concatenate([np.array(probes, np.float32), rng.uniform(-1, 1, 100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, -1.0], np.float32)])
    assert np.array_equal(nf4.nearest_code(n, lv), nf4.nearest_code_fast(n, lv))
