"""Oracle: blockwise NF4 quantization with double quantization (CPU, numpy).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Every step follows the
pages' description in their order; where the pages are silent the reading used
is stated at the function.

Data layout (the same contract the CUDA library implements independently):
  * W is taken as one flat row-major sequence of ``numel`` fp32 values.
  * block  = 64 consecutive flat elements (last block may be partial);
  * group  = 256 consecutive blocks (last group may be partial);
  * codes  = ceil(numel/2) bytes, flat element 2j in the LOW nibble of byte j,
             element 2j+1 in the HIGH nibble; an unused final high nibble is 0;
  * absmax_q    = one uint8 per block (the int8 bit pattern in the signed
                  double-quantization variant);
  * group_scale = one fp32 per group;
  * offset      = the signed variant's tensor-wide mean block constant (fp32).

Precision: all scalar steps are IEEE fp32 round-to-nearest-even (numpy float32
arithmetic, no fused multiply-add), written ``fl32(.)`` below; bf16(.) is
fp32 -> bf16 round-to-nearest-even.
"""

from __future__ import annotations

import math

import numpy as np
import mpmath

BLOCK = 64          # weights per absmax block
GROUP = 256         # blocks per double-quantization group
NLEVELS = 16


# ---------------------------------------------------------------------------
# Codebook
# ---------------------------------------------------------------------------

def nf4_levels_exact(dps: int = 50):
    """The 16 NF4 levels as high-precision mpmath numbers, ascending.

    [Blog-nf4]: the 16 NF4 levels sit at normal quantiles, so for Gaussian
    weights every level is hit about equally often; [QLoRA-abs] (a): the type
    is designed to be optimal for normally distributed weights;
    [Cap-nf4]: combined with block-wise absmax scaling.

    Reading (the pages give no formula): the levels must span [-1, 1] (absmax
    scaling maps every block into that interval) and contain an exact zero (so
    a zero weight and an all-zero block survive).  16 = 1 zero + 8 positive +
    7 negative quantiles.  The positive levels are the standard-normal
    quantiles Phi^-1(p) at the 8 points p = d + (1/2 - d) i / 8, i = 0..7, the
    negative ones are -Phi^-1(p) at p = d + (1/2 - d) i / 7, i = 0..6, with the
    outer probability d = 1 - (1/32 + 1/30)/2 (finite quantile at the edge,
    the midpoint of the 1/32 and 1/30 tail masses of 16 and 15 equal slices).
    The set is divided by its largest magnitude so both ends land on +-1.
    """
    mp = mpmath.mp.clone()
    mp.dps = dps
    d = 1 - (mp.mpf(1) / 32 + mp.mpf(1) / 30) / 2

    def phi_inv(p):
        return mp.sqrt(2) * mp.erfinv(2 * p - 1)

    pos = [phi_inv(d + (mp.mpf(1) / 2 - d) * i / 8) for i in range(8)]
    neg = [-phi_inv(d + (mp.mpf(1) / 2 - d) * i / 7) for i in range(7)]
    vals = sorted(pos + neg + [mp.mpf(0)])
    top = max(abs(v) for v in vals)
    return [v / top for v in vals]


FORMATS = ("nf4", "fp4", "int4")


def fp4_codebook() -> np.ndarray:
    """Plain 4-bit float ([Blog-nf4] / [Cap-qlora] name it only as the weaker
    alternative; reading: the e2m1 layout, 1 sign, 2 exponent, 1 mantissa bit,
    magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6) scaled by 1/6 so the largest level is
    1.  Codes 0..7 hold -1 .. -0 ascending, codes 8..15 hold +0 .. +1.  The two
    zeros are equal, so nearest-level encoding with ties to the lower index
    never emits code 8."""
    mag = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float32)
    pos = (mag / np.float32(6.0)).astype(np.float32)
    neg = (-mag[::-1] / np.float32(6.0)).astype(np.float32)   # -1 .. -0 (the last one is -0.0)
    return np.concatenate([neg, pos]).astype(np.float32)


def int4_codebook() -> np.ndarray:
    """Plain 4-bit integer grid ([Blog-nf4]: NF4 beats plain integer types;
    reading: symmetric absmax scaling, the block maximum maps to 7):
    level[c] = fl32((c - 8) / 7), c = 0..15 (level[0] = -8/7 is never the
    nearest level of a normalised value in [-1, 1])."""
    c = np.arange(16, dtype=np.float32)
    return ((c - np.float32(8.0)) / np.float32(7.0)).astype(np.float32)


def codebook(fmt: str = "nf4") -> np.ndarray:
    """The 16 ascending fp32 levels of a 4-bit table."""
    if fmt == "nf4":
        return nf4_codebook()
    if fmt == "fp4":
        return fp4_codebook()
    if fmt == "int4":
        return int4_codebook()
    raise ValueError(fmt)


def nf4_codebook() -> np.ndarray:
    """The 16 levels rounded to fp32 (round-to-nearest), ascending."""
    return np.array([float(v) for v in nf4_levels_exact()], dtype=np.float64).astype(np.float32)


# ---------------------------------------------------------------------------
# bf16 helpers (bit patterns carried as uint16)
# ---------------------------------------------------------------------------

def bf16_rne_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 round-to-nearest-even, returned as uint16 bit patterns.

    Definition: keep the upper 16 bits of the fp32 pattern, rounding the
    discarded 16 bits to nearest with ties to an even kept part.  Inputs must be
    finite (the quantizer rejects non-finite weights).
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    keep = u >> 16
    rest = u & 0xFFFF
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & 1) == 1))
    return (keep + up.astype(np.uint64)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# Quantization steps
# ---------------------------------------------------------------------------

def num_blocks(numel: int) -> int:
    return -(-numel // BLOCK)


def num_groups(numel: int) -> int:
    return -(-num_blocks(numel) // GROUP)


def footprint_bytes(numel: int) -> int:
    """Bytes of the packed representation: codes + u8 constants + fp32 scales."""
    return -(-numel // 2) + num_blocks(numel) + 4 * num_groups(numel)


def block_absmax(w_flat: np.ndarray) -> np.ndarray:
    """a_b = max |w| over each block of 64 consecutive flat elements (fp32, exact).

    [Blog-nf4] (one scaling constant per block of weights), [Cap-nf4]
    (block-wise absmax scaling), [Cap-qlora] (absmax tracking).
    """
    w = np.asarray(w_flat, dtype=np.float32).ravel()
    nb = num_blocks(w.size)
    pad = nb * BLOCK - w.size
    a = np.abs(w)
    if pad:
        a = np.concatenate([a, np.zeros(pad, np.float32)])
    return a.reshape(nb, BLOCK).max(axis=1).astype(np.float32)


def normalize(w_flat: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """n = fl32(w / a_b) for each element; n = 0 where a_b = 0 (all-zero block)."""
    w = np.asarray(w_flat, dtype=np.float32).ravel()
    a = np.repeat(absmax, BLOCK)[: w.size]
    n = np.zeros_like(w)
    nz = a != 0
    n[nz] = w[nz] / a[nz]          # float32 / float32: IEEE RN
    return n


def nearest_code(n: np.ndarray, levels: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """code = argmin_i |n - v_i| with ties broken to the LOWER index.

    Distances are taken in fp64; for fp32 n and fp32 levels they are exact
    wherever two distances can be close to a tie (every midpoint between
    adjacent levels has magnitude >= 0.039), so the argmin is exact.
    numpy's argmin returns the first minimum, i.e. the lower index.
    """
    n = np.asarray(n, dtype=np.float32).ravel()
    v = np.asarray(levels, dtype=np.float32).astype(np.float64)
    out = np.empty(n.size, dtype=np.uint8)
    for s in range(0, n.size, chunk):
        x = n[s:s + chunk].astype(np.float64)
        dist = np.abs(x[:, None] - v[None, :])
        out[s:s + chunk] = np.argmin(dist, axis=1).astype(np.uint8)
    return out


def nearest_code_fast(n: np.ndarray, levels: np.ndarray) -> np.ndarray:
    """The same code as nearest_code (nearest level, ties to the lower index),
    for large inputs: with ascending levels, the nearest level of n is the
    number of midpoints strictly below n, each midpoint of two fp32 levels
    being exact in fp64; between two equal levels the upper one is never
    strictly nearer, so that midpoint is skipped.  Equality with the argmin
    definition is checked by the tests on dense probes around every midpoint."""
    v = np.asarray(levels, dtype=np.float32).astype(np.float64)
    mids = [(v[i] + v[i + 1]) / 2 for i in range(len(v) - 1) if v[i] != v[i + 1]]
    skip = [i for i in range(len(v) - 1) if v[i] == v[i + 1]]
    x = np.asarray(n, dtype=np.float32).ravel().astype(np.float64)
    k = np.searchsorted(np.array(mids), x, side="left")     # midpoints strictly below x
    # map the count over distinct-level midpoints back to a code index
    code_of = []
    c = 0
    for i in range(len(v) - 1):
        if i in skip:
            continue
        code_of.append(c)
        c = i + 1
    code_of.append(c)
    return np.asarray(code_of, dtype=np.uint8)[k]


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2j -> low nibble, 2j+1 -> high nibble."""
    c = np.asarray(codes, dtype=np.uint8).ravel()
    if c.size % 2:
        c = np.concatenate([c, np.zeros(1, np.uint8)])
    return (c[0::2] & 0xF) | ((c[1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray, numel: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).ravel()
    c = np.empty(p.size * 2, dtype=np.uint8)
    c[0::2] = p & 0xF
    c[1::2] = p >> 4
    return c[:numel]


def double_quantize(absmax: np.ndarray):
    """Quantize the fp32 block constants to 8 bits with one fp32 scale per group.

    [Blog-nf4] (double quantization stores the per-block constants in 8-bit
    under one more, coarser level of constants), [QLoRA-abs] (b),
    [Cap-nf4].  Reading (the 8-bit format is not given): unsigned linear
    8-bit codes with no offset, group = 256 consecutive blocks:
        c_g = max_b a_b,   S_g = fl32(c_g / 255),
        q_b = min(255, round_half_even(fl32(a_b / S_g)))   (q_b = 0 if S_g == 0).
    Returns (q uint8 [nblocks], S float32 [ngroups]).
    """
    a = np.asarray(absmax, dtype=np.float32).ravel()
    nb = a.size
    ng = -(-nb // GROUP)
    pad = ng * GROUP - nb
    ap = np.concatenate([a, np.zeros(pad, np.float32)]) if pad else a
    c = ap.reshape(ng, GROUP).max(axis=1).astype(np.float32)
    S = (c / np.float32(255.0)).astype(np.float32)
    Sb = np.repeat(S, GROUP)[:nb]
    q = np.zeros(nb, dtype=np.uint8)
    nz = Sb != 0
    ratio = (a[nz] / Sb[nz]).astype(np.float32)           # fl32(a_b / S_g)
    r = np.rint(ratio)                                      # half-to-even
    q[nz] = np.minimum(r, 255.0).astype(np.uint8)
    return q, S


def dequantize_absmax(q: np.ndarray, S: np.ndarray) -> np.ndarray:
    """a'_b = fl32(q_b * S_g)."""
    q = np.asarray(q, dtype=np.uint8).ravel()
    Sb = np.repeat(np.asarray(S, np.float32), GROUP)[: q.size]
    return (q.astype(np.float32) * Sb).astype(np.float32)


# ---------------------------------------------------------------------------
# Double quantization, variant with a tensor-wide offset and signed codes
# ---------------------------------------------------------------------------
#
# The pages say only that the block constants are stored in 8 bits under a
# coarser set of constants ([Blog-nf4], [QLoRA-abs] (b), [Cap-nf4] "nested
# quantization").  The variant below is a second reading of that sentence:
# the block constants of a tensor are all positive and cluster around their
# mean, so the mean is taken out first and the 8-bit code only carries the
# signed deviation from it.  Every step is fixed so that the result does not
# depend on any summation order:
#
#   mu   = fl32( fl64( fl64(sum_b a_b) / n_blocks ) )   sum_b a_b exact
#   c_b  = fl32(a_b - mu)
#   S_g  = fl32( max_{b in g} |c_b| / 127 )
#   q_b  = clamp(round_half_even(fl32(c_b / S_g)), -127, 127)   (0 if S_g == 0)
#   a'_b = fl32( fl32(q_b * S_g) + mu )
#
# fl64(.) is round-to-nearest-even to binary64.  The codes are stored as the
# int8 bit patterns of q_b; -128 is never produced.

F32_MIN_EXP = -149          # exponent of the smallest fp32 subnormal


def exact_sum_units(a: np.ndarray) -> int:
    """sum_b a_b exactly, as an integer count of 2^-149 units.

    Every finite fp32 value is an integer multiple of 2^-149, so the sum of
    non-negative fp32 values is an integer in those units; Python integers hold
    it without rounding.  a * 2^149 is exact in fp64 (a power-of-two scaling
    inside fp64's range) and int() of an integral fp64 value is exact."""
    a64 = np.asarray(a, dtype=np.float32).astype(np.float64).ravel()
    if np.any(a64 < 0):
        raise ValueError("block constants are non-negative")
    scaled = np.ldexp(a64, -F32_MIN_EXP)
    return sum(int(x) for x in scaled.tolist())


def block_constant_mean(a: np.ndarray) -> np.float32:
    """mu = fl32(fl64(fl64(exact sum) / n)): the tensor-wide mean block constant.

    float() of a Python int rounds to nearest-even; ldexp by -149 is exact
    (the sum of fp32 values is far inside fp64's normal range); the fp64
    division is IEEE round-to-nearest-even; np.float32() rounds once more."""
    n = int(np.asarray(a).size)
    if n == 0:
        return np.float32(0.0)
    s64 = math.ldexp(float(exact_sum_units(a)), F32_MIN_EXP)
    return np.float32(s64 / float(n))


def double_quantize_signed(absmax: np.ndarray):
    """Signed 8-bit block constants around the tensor-wide mean (see above).

    Returns (q uint8 [nblocks] holding int8 bit patterns, S float32 [ngroups],
    mu float32)."""
    a = np.asarray(absmax, dtype=np.float32).ravel()
    nb = a.size
    ng = -(-nb // GROUP)
    mu = block_constant_mean(a)
    c = (a - mu).astype(np.float32)                         # fl32(a_b - mu)
    pad = ng * GROUP - nb
    cp = np.concatenate([c, np.zeros(pad, np.float32)]) if pad else c
    m = np.abs(cp).reshape(ng, GROUP).max(axis=1).astype(np.float32)
    S = (m / np.float32(127.0)).astype(np.float32)
    Sb = np.repeat(S, GROUP)[:nb]
    q = np.zeros(nb, dtype=np.int8)
    nz = Sb != 0
    ratio = (c[nz] / Sb[nz]).astype(np.float32)            # fl32(c_b / S_g)
    q[nz] = np.clip(np.rint(ratio), -127.0, 127.0).astype(np.int8)
    return q.view(np.uint8), S, mu


def dequantize_absmax_signed(q: np.ndarray, S: np.ndarray, mu) -> np.ndarray:
    """a'_b = fl32(fl32(q_b * S_g) + mu), q_b the int8 value of the stored byte."""
    qi = np.asarray(q, dtype=np.uint8).ravel().view(np.int8)
    Sb = np.repeat(np.asarray(S, np.float32), GROUP)[: qi.size]
    return ((qi.astype(np.float32) * Sb).astype(np.float32) + np.float32(mu)).astype(np.float32)


DQ_VARIANTS = ("plain", "signed")


def quantize_nf4(W: np.ndarray, fmt: str = "nf4", dq: str = "plain"):
    """Quantize fp32 weights once, up front ([Blog-mem]: the base never changes,
    so it is quantized once).

    Steps in the pages' order: block absmax -> normalise -> nearest NF4 level
    -> pack 4-bit codes -> double-quantize the block constants.  The codes use
    the exact fp32 block absmax (the constants are quantized afterwards, as a
    separate second level).  dq picks the reading of the second level:
    "plain" (double_quantize) or "signed" (double_quantize_signed).  Raises
    ValueError on non-finite input.

    Returns dict(codes=uint8[ceil(numel/2)], absmax_q=uint8[nblocks],
    group_scale=float32[ngroups], offset=float32 (mu; 0 for "plain"),
    shape=W.shape, format=fmt, dq=dq).
    """
    if dq not in DQ_VARIANTS:
        raise ValueError(f"unknown double-quantization variant {dq!r}")
    W = np.asarray(W, dtype=np.float32)
    if not np.all(np.isfinite(W)):
        raise ValueError("non-finite weight")
    flat = W.ravel()
    a = block_absmax(flat)
    n = normalize(flat, a)
    codes = nearest_code(n, codebook(fmt)) if n.size <= (1 << 24) else nearest_code_fast(n, codebook(fmt))
    if dq == "plain":
        q, S = double_quantize(a)
        mu = np.float32(0.0)
    else:
        q, S, mu = double_quantize_signed(a)
    return {"codes": pack_nibbles(codes), "absmax_q": q, "group_scale": S, "offset": mu,
            "shape": tuple(W.shape), "format": fmt, "dq": dq}


def dequantize_nf4_bits(codes: np.ndarray, absmax_q: np.ndarray, group_scale: np.ndarray,
                        shape, fmt: str = "nf4", dq: str = "plain", offset=0.0) -> np.ndarray:
    """W' = bf16(fl32(v_code * a'_b)); bf16 bit patterns.  a'_b = fl32(q_b * S_g)
    for the plain constants, fl32(fl32(q_b * S_g) + mu) for the signed ones.

    [Blog-mem]: every forward and backward pass expands the 4-bit base back
    to a 16-bit type as it runs.  Reading: the 16-bit type is bf16, the product
    is formed in fp32 then rounded once to bf16.
    """
    numel = int(np.prod(shape))
    c = unpack_nibbles(codes, numel)
    v = codebook(fmt)[c]
    if dq == "plain":
        a_deq = dequantize_absmax(absmax_q, group_scale)
    else:
        a_deq = dequantize_absmax_signed(absmax_q, group_scale, offset)
    ap = np.repeat(a_deq, BLOCK)[:numel]
    w32 = (v * ap).astype(np.float32)
    return bf16_rne_bits(w32).reshape(shape)


def dequantize_nf4(q: dict) -> np.ndarray:
    """Convenience: dequantize a quantize_nf4() result to bf16 bit patterns."""
    return dequantize_nf4_bits(q["codes"], q["absmax_q"], q["group_scale"], q["shape"], q.get("format", "nf4"),
                               q.get("dq", "plain"), q.get("offset", 0.0))


def reconstruction_error(W: np.ndarray, fmt: str = "nf4", dq: str = "plain") -> float:
    """Relative Frobenius error ||bf16 dequant(quant(W)) - W|| / ||W|| of a 4-bit
    table on the given weights: the proxy, on Gaussian weights, for the pages'
    statement that NF4 beats plain 4-bit float and integer types ([Blog-nf4])."""
    W = np.asarray(W, dtype=np.float32)
    Wd = bf16_bits_to_f32(dequantize_nf4(quantize_nf4(W, fmt, dq))).astype(np.float64)
    W64 = W.astype(np.float64)
    return float(np.linalg.norm(Wd - W64) / np.linalg.norm(W64))
