"""The plain 4-bit float and integer tables through every kernel: quantizer
and dequantizer bit-exact against the oracle, and the linear forward and
backward (few-token kernel, one-CTA and CTA-pair GEMMs) within the parity
tolerance, for FP4 and Int4."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from oracle import nf4 as onf4
from tests.gpu_util import TOL, f64, rel

pytestmark = pytest.mark.gpu

FMTS = {"fp4": q.FORMAT_FP4, "int4": q.FORMAT_INT4}


def _weights(W, fmt):
    oq = onf4.quantize_nf4(W.numpy(), fmt)
    w = q.quantize_nf4(W.cuda().contiguous(), format=FMTS[fmt])
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert np.array_equal(w.codes.cpu().numpy(), oq["codes"])
    assert np.array_equal(w.absmax_q.cpu().numpy(), oq["absmax_q"])
    assert np.array_equal(w.group_scale.cpu().numpy().view(np.uint32), oq["group_scale"].view(np.uint32))
    return w, oq


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("shape", [(256, 1024), (3, 16384 + 64 * 5 + 7), (1032, 4160)])
def test_quantize_dequantize_bit_exact(lib, fmt, shape):
    W = qi.make_weight(*shape, seed=50 + shape[0])
    W[0, :64] = 0.0                       # an all-zero block: every code is the table's zero
    w, oq = _weights(W, fmt)
    got = q.dequantize(w).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, onf4.dequantize_nf4(oq))
    if fmt == "fp4":
        codes = onf4.unpack_nibbles(oq["codes"], W.numel())
        assert not np.any(codes == 8)


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("M,N,K,r", [(1, 776, 2112, 24), (12, 520, 704, 16), (96, 512, 448, 64),
                                     (300, 1032, 1152, 32)])
def test_linear_parity(lib, fmt, M, N, K, r):
    case = qi.LinearCase(f"{fmt}_{M}_{N}_{K}_{r}", M, N, K, r, 16.0, 500 + M + N + K + r)
    d = qi.make_linear(case)
    w, oq = _weights(d["W"], fmt)
    Wd = onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd(w, X, A, B, d["s"])
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    Yr, Hr = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    dXr, dAr, dBr = olin.lora_linear_bwd(Wd, f64(d["X"]), f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
    errs = {"Y": rel(f64(Y), Yr), "H": rel(f64(H), Hr), "dX": rel(f64(dX), dXr), "dA": rel(f64(dA), dAr),
            "dB": rel(f64(dB), dBr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)


def test_reconstruction_error_on_the_gpu(lib):
    """The same proxy as the oracle's, through the library: NF4 beats FP4 and
    Int4 on Gaussian weights, and each error equals the oracle's."""
    W = qi.make_weight(1024, 4096, seed=61)
    err = {}
    for fmt, fid in (("nf4", q.FORMAT_NF4), ("fp4", q.FORMAT_FP4), ("int4", q.FORMAT_INT4)):
        w = q.quantize_nf4(W.cuda(), format=fid)
        Wd = q.dequantize(w).float().cpu().numpy().astype(np.float64)
        W64 = W.numpy().astype(np.float64)
        err[fmt] = float(np.linalg.norm(Wd - W64) / np.linalg.norm(W64))
        assert err[fmt] == pytest.approx(onf4.reconstruction_error(W.numpy(), fmt), rel=1e-12)
    assert err["nf4"] < err["fp4"] and err["nf4"] < err["int4"], err
