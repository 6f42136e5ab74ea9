"""The C-ABI library loads, exports every declared symbol, and validates
arguments on the host (no GPU needed: every call here returns before any CUDA
work is enqueued)."""

import ctypes
import os
import re

import numpy as np
import pytest

import bit_quantized_lora_nf4_b200 as q
from oracle import nf4

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "qlora.h")


def _declared():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    txt = re.sub(r"typedef[^;]*;", "", txt)         # function-pointer types are not exports
    return sorted(set(re.findall(r"\b(qlora_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = q.load()
    decl = _declared()
    assert len(decl) >= 13
    for name in decl:
        assert hasattr(lib, name), name
    assert sorted(q.EXPORTS) == decl


def test_codebook_matches_oracle_bitwise():
    lib_cb = np.array(q.codebook(), dtype=np.float32)
    assert np.array_equal(lib_cb.view(np.uint32), nf4.nf4_codebook().view(np.uint32))


def test_size_helpers():
    lib = q.load()
    for rows, cols in ((256, 256), (4096, 11008), (3, 5), (1, 1)):
        n = rows * cols
        assert lib.qlora_codes_bytes(rows, cols) == (n + 1) // 2
        assert lib.qlora_absmax_bytes(rows, cols) == nf4.num_blocks(n)
        assert lib.qlora_group_scale_bytes(rows, cols) == 4 * nf4.num_groups(n)
        assert (lib.qlora_codes_bytes(rows, cols) + lib.qlora_absmax_bytes(rows, cols)
                + lib.qlora_group_scale_bytes(rows, cols)) == nf4.footprint_bytes(n)


def test_status_strings():
    lib = q.load()
    for code, name in q.STATUS_NAMES.items():
        assert lib.qlora_status_string(code).decode() == name


def test_workspace_sizes_positive_and_monotone():
    for op in (q.QLORA_OP_FWD, q.QLORA_OP_BWD):
        a = q.workspace_bytes(op, 4096, 4096, 4096, 64)
        b = q.workspace_bytes(op, 8192, 4096, 4096, 64)
        assert 256 <= a <= b
    assert q.workspace_bytes(7, 1, 1, 1, 1) == 0


def test_stream_k_mode_round_trip():
    lib = q.load()
    assert lib.qlora_set_stream_k(q.STREAM_K_ALWAYS) == q.STREAM_K_AUTO       # the default
    assert lib.qlora_set_stream_k(q.STREAM_K_OFF) == q.STREAM_K_ALWAYS
    assert lib.qlora_set_stream_k(3) == -1 and lib.qlora_set_stream_k(-1) == -1
    assert q.set_stream_k(q.STREAM_K_AUTO) == q.STREAM_K_OFF
    with pytest.raises(ValueError):
        q.set_stream_k(7)


def test_stream_k_region_is_an_optional_tail():
    """The fused GEMMs' stream-K pieces are the last, optional part of the
    workspace: present for the CTA-pair kernel (M > 128, or a dense weight),
    at most 2 x 2 x 80 fp32 tile pieces of 128 x 256 x NACC per CTA, absent for the
    few-token and one-CTA paths."""
    lib = q.load()
    piece = 128 * 256 * 4
    for op in range(4):
        for M, nacc in ((4096, 2), (300, 2), (200, 1)):
            full = lib.qlora_workspace_bytes(op, M, 4096, 4096, 64)
            low = lib.qlora_workspace_min_bytes(op, M, 4096, 4096, 64)
            assert 256 <= low < full
            assert full - low >= 80 * 2 * 2 * nacc * piece
            assert full - low <= 80 * 2 * 2 * nacc * piece + 4096
    for op in (q.QLORA_OP_FWD, q.QLORA_OP_BWD):
        for M in (1, 16, 128):     # few-token or one-CTA kernels: no tail
            assert lib.qlora_workspace_min_bytes(op, M, 4096, 4096, 64) == lib.qlora_workspace_bytes(op, M, 4096, 4096, 64)
    for op in (q.QLORA_OP_FWD_DENSE, q.QLORA_OP_BWD_DENSE):
        assert lib.qlora_workspace_min_bytes(op, 16, 4096, 4096, 64) < lib.qlora_workspace_bytes(op, 16, 4096, 4096, 64)
    assert lib.qlora_workspace_min_bytes(9, 1, 1, 1, 1) == 0
    # below the minimum the calls refuse, with nothing launched
    for op, call in ((q.QLORA_OP_FWD, _fwd), (q.QLORA_OP_BWD, _bwd)):
        ws_min = lib.qlora_workspace_min_bytes(op, 4096, 4096, 4096, 64)
        assert call(_w(4096, 4096), M=4096, r=64, wsb=ws_min - 1) == 7


# ---------------------------------------------------------------- host-side argument errors

FAKE = 0x10000          # 16-byte aligned, never dereferenced: validation fails first
MIS = 0x10001           # misaligned


def _w(rows=256, cols=256, codes=FAKE, absmax=FAKE, scale=FAKE):
    return q.Nf4WeightC(rows, cols, codes, absmax, scale)


def _fwd(w, X=FAKE, M=64, A=FAKE, B=FAKE, r=16, s=1.0, Y=FAKE, H=None, ws=FAKE, wsb=1 << 40):
    lib = q.load()
    return lib.qlora_linear_fwd(ctypes.byref(w), X, M, A, B, r, s, Y, H, ws, wsb, None)


def _bwd(w, X=FAKE, dY=FAKE, M=64, A=FAKE, B=FAKE, r=16, s=1.0, dX=FAKE, dA=FAKE, dB=FAKE, ws=FAKE, wsb=1 << 40):
    lib = q.load()
    return lib.qlora_linear_bwd(ctypes.byref(w), X, dY, M, A, B, r, s, None, dX, dA, dB, ws, wsb, None)


def test_linear_argument_errors():
    assert _fwd(_w(codes=None)) == 1
    assert _fwd(_w(), X=None) == 1
    assert _fwd(_w(), M=0) == 1
    assert _fwd(_w(), r=4) == 1
    assert _fwd(_w(), r=512) == 1
    assert _fwd(_w(), s=float("nan")) == 1
    assert _fwd(_w(), r=20) == 2                     # r % 8
    assert _fwd(_w(cols=200)) == 2                   # K % 64
    assert _fwd(_w(rows=250)) == 2                   # N % 8
    assert _fwd(_w(), X=MIS) == 3
    assert _fwd(_w(absmax=MIS)) == 3
    assert _fwd(_w(), wsb=16) == 7
    assert _fwd(_w(), ws=None) == 7
    assert _bwd(_w(), dY=None) == 1
    assert _bwd(_w(), dA=MIS) == 3
    assert _bwd(_w(), wsb=0) == 7


def test_quantize_dequantize_argument_errors():
    lib = q.load()
    w = _w()
    for dt in (q.DTYPE_F32, q.DTYPE_BF16):
        assert lib.qlora_quantize_nf4(None, dt, ctypes.byref(w), None) == 1
        assert lib.qlora_quantize_nf4(MIS, dt, ctypes.byref(w), None) == 3
        assert lib.qlora_quantize_nf4(FAKE, dt, ctypes.byref(_w(rows=0)), None) == 1
    # element types other than fp32 / bf16 are refused before anything is enqueued
    for dt in (-1, 2, 7):
        assert lib.qlora_quantize_nf4(FAKE, dt, ctypes.byref(w), None) == 1
        assert lib.qlora_quantize_nf4_ws(FAKE, dt, ctypes.byref(w), FAKE, 1 << 20, None) == 1
    assert lib.qlora_dequantize(ctypes.byref(w), None, None) == 1
    assert lib.qlora_dequantize(ctypes.byref(_w(scale=MIS)), FAKE, None) == 3
    assert lib.qlora_nf4_codebook(None) == 1


def test_wait_limit_roundtrip():
    old = q.set_wait_limit(12345)
    assert q.set_wait_limit(old) == 12345


def test_signed_block_constant_sizes_and_errors():
    lib = q.load()
    for rows, cols in ((256, 256), (4096, 11008), (3, 5)):
        n = rows * cols
        assert lib.qlora_group_scale_bytes_dq(rows, cols, q.DQ_PLAIN) == 4 * nf4.num_groups(n)
        assert lib.qlora_group_scale_bytes_dq(rows, cols, q.DQ_SIGNED) == 4 * nf4.num_groups(n) + 4
        assert lib.qlora_quantize_workspace_bytes(rows, cols, q.DQ_PLAIN) == 0
        ws = lib.qlora_quantize_workspace_bytes(rows, cols, q.DQ_SIGNED)
        assert ws % 256 == 0 and ws >= 128 + 4 * nf4.num_blocks(n)
    assert lib.qlora_group_scale_bytes_dq(4, 4, 2) == 0
    w = q.Nf4WeightC(256, 256, FAKE, FAKE, FAKE, q.FORMAT_NF4, q.DQ_SIGNED)
    assert lib.qlora_quantize_nf4(FAKE, q.DTYPE_F32, ctypes.byref(w), None) == 7          # needs the workspace call
    assert lib.qlora_quantize_nf4_ws(FAKE, q.DTYPE_BF16, ctypes.byref(w), FAKE, 16, None) == 7
    assert lib.qlora_quantize_nf4_ws(FAKE, q.DTYPE_F32, ctypes.byref(w), MIS, 1 << 20, None) == 3
    big = q.Nf4WeightC(1 << 20, 1 << 18, FAKE, FAKE, FAKE, q.FORMAT_NF4, q.DQ_SIGNED)
    assert lib.qlora_quantize_nf4_ws(FAKE, q.DTYPE_F32, ctypes.byref(big), FAKE, 1 << 62, None) == 2
    bad = q.Nf4WeightC(256, 256, FAKE, FAKE, FAKE, q.FORMAT_NF4, 2)
    assert lib.qlora_quantize_nf4(FAKE, q.DTYPE_F32, ctypes.byref(bad), None) == 1
    assert lib.qlora_dequantize(ctypes.byref(bad), FAKE, None) == 1
    assert _fwd(bad) == 1


def test_lq_sizes_and_argument_errors():
    lib = q.load()
    assert lib.qlora_lq_workspace_bytes(256, 512, 16, 24, 0) >= 4 * 256 * 512
    assert lib.qlora_lq_workspace_bytes(256, 512, 16, 0, 0) > 0          # residual quantizer alone
    assert lib.qlora_lq_workspace_bytes(256, 512, 16, 8, 0) == 0         # l < r
    assert lib.qlora_lq_workspace_bytes(256, 512, 16, 98, 0) == 0        # l > 96
    assert lib.qlora_lq_workspace_bytes(256, 512, 16, 24, 5) == 0        # unknown dq
    w = q.Nf4WeightC(256, 512, FAKE, FAKE, FAKE, 0, 0)
    big = 1 << 40

    def dec(W=FAKE, Q=w, L1=FAKE, L2=FAKE, r=16, Om=FAKE, l=24, power=2, iters=2, err=FAKE, ws=FAKE, wsb=big):
        return lib.qlora_lq_decompose(W, ctypes.byref(Q), L1, L2, r, Om, l, power, iters, err, ws, wsb, None)
    assert dec(W=None) == 1
    assert dec(err=None) == 1
    assert dec(l=23) == 1                      # odd test-matrix width
    assert dec(l=8) == 1                       # l < r
    assert dec(iters=0) == 1
    assert dec(power=-1) == 1
    assert dec(Q=q.Nf4WeightC(20, 512, FAKE, FAKE, FAKE, 0, 0)) == 2      # fewer rows than l
    assert dec(wsb=1024) == 7
    assert dec(W=MIS) == 3
    assert dec(Om=MIS) == 3
    assert lib.qlora_lq_lowrank(FAKE, 256, 512, ctypes.byref(q.Nf4WeightC(256, 256, FAKE, FAKE, FAKE, 0, 0)),
                                FAKE, 24, 2, 16, FAKE, FAKE, FAKE, big, None) == 1       # shape mismatch
    assert lib.qlora_lq_lowrank(FAKE, 10, 512, None, FAKE, 24, 2, 16, FAKE, FAKE, FAKE, big, None) == 2
    assert lib.qlora_lq_lowrank(FAKE, 256, 512, None, FAKE, 26, 2, 16, FAKE, FAKE, FAKE, big, None) == 1   # l % 4
    assert lib.qlora_lq_quantize_residual(FAKE, None, FAKE, 16, ctypes.byref(w), FAKE, big, None) == 1
    assert lib.qlora_lq_quantize_residual(FAKE, FAKE, FAKE, 16, ctypes.byref(w), FAKE, 64, None) == 7


def test_dense_linear_sizes_and_argument_errors():
    lib = q.load()
    for op in (q.QLORA_OP_FWD_DENSE, q.QLORA_OP_BWD_DENSE):
        assert lib.qlora_workspace_bytes(op, 4, 512, 512, 16) >= 256
    assert lib.qlora_workspace_bytes(4, 4, 512, 512, 16) == 0
    big = 1 << 40
    f = lib.qlora_linear_fwd_dense
    assert f(None, 256, 256, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, big, None) == 1
    assert f(FAKE, 256, 200, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, big, None) == 2     # K % 64
    assert f(MIS, 256, 256, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, big, None) == 3
    assert f(FAKE, 256, 256, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, 16, None) == 7
    b = lib.qlora_linear_bwd_dense
    assert b(FAKE, 256, 256, FAKE, None, 64, FAKE, FAKE, 16, 1.0, None, FAKE, FAKE, FAKE, FAKE, big, None) == 1
    calls = []

    def cb(ctx, w_out, n, k, stream):
        calls.append((n, k))
        return 0
    fn = q.MATERIALIZE_FN(cb)
    m = lib.qlora_linear_fwd_materialized
    assert m(fn, None, FAKE, 256, 200, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, big, None) == 2
    assert m(fn, None, FAKE, 256, 256, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, 16, None) == 7
    assert calls == []          # argument errors are found before the weight is materialized
    bad = q.MATERIALIZE_FN(lambda ctx, w_out, n, k, stream: 4)
    assert m(bad, None, FAKE, 256, 256, FAKE, 64, FAKE, FAKE, 16, 1.0, FAKE, None, FAKE, big, None) == 4


def test_noalloc_scratch_size_and_documented_limits():
    """The binding's copy of QLORA_STATIC_SCRATCH_BYTES matches the header, and
    the size limits the header states for qlora_linear_fwd_noalloc hold for the
    library's own workspace sizing (host-only calls)."""
    hdr = open(HEADER).read()
    m = re.search(r"#define QLORA_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == q.QLORA_STATIC_SCRATCH_BYTES
    lib = q.load()
    lim = q.QLORA_STATIC_SCRATCH_BYTES
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008), (8192, 22016)):
        assert lib.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 2048, N, K, 64) <= lim
        assert lib.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 3413, N, K, 64) <= lim
        assert lib.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 3414, N, K, 64) > lim
        assert lib.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 862, N, K, 256) <= lim
        assert lib.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 863, N, K, 256) > lim
        # the stream-K tail never fits beside the forward
        assert lib.qlora_workspace_bytes(q.QLORA_OP_FWD, 256, N, K, 64) > lim


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checked debug build (built beside the release library) loads
    and exports the same C ABI."""
    assert os.path.exists(q.DEBUG_LIB_PATH), "libqlora_debug.so not built"
    dbg = ctypes.CDLL(q.DEBUG_LIB_PATH)
    for name in _declared():
        assert hasattr(dbg, name), name
    dbg.qlora_status_string.restype = ctypes.c_char_p
    assert dbg.qlora_status_string(8).decode() == "QLORA_ERR_BOUNDS"
