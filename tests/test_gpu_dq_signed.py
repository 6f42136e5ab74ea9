"""Signed block constants around the tensor-wide mean (QLORA_DQ_SIGNED)
through every kernel: quantizer (codes, int8 constants, group scales and the
offset mu) and dequantizer bit-exact against the oracle; mu independent of
the order of the blocks; the linear forward and backward (few-token kernel,
one-CTA and CTA-pair GEMMs, with padded rows and blocks) within the parity
tolerance; NF4 and FP4 tables."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from oracle import nf4 as onf4
from tests.gpu_util import TOL, f64, rel

pytestmark = pytest.mark.gpu

FMTS = {"nf4": q.FORMAT_NF4, "fp4": q.FORMAT_FP4}


def _signed(W, fmt="nf4"):
    oq = onf4.quantize_nf4(W.numpy(), fmt, dq="signed")
    w = q.quantize_nf4(W.cuda().contiguous(), format=FMTS[fmt], dq=q.DQ_SIGNED)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert np.array_equal(w.codes.cpu().numpy(), oq["codes"]), "codes differ"
    assert np.array_equal(w.absmax_q.cpu().numpy(), oq["absmax_q"]), "int8 constants differ"
    assert np.array_equal(w.scales.cpu().numpy().view(np.uint32), oq["group_scale"].view(np.uint32)), "scales differ"
    assert w.offset.cpu().numpy().view(np.uint32)[0] == np.float32(oq["offset"]).view(np.uint32), "mu differs"
    return w, oq


def _awkward_weight(rows, cols, seed):
    """Gaussian weights with an all-zero block, a block of outliers, a region
    at a tiny scale and a constant block (some groups far from the mean)."""
    W = qi.make_weight(rows, cols, seed=seed)
    flat = W.view(-1)
    flat[:64] = 0.0
    flat[64 * 5:64 * 6] *= 40.0
    n = flat.numel()
    flat[n // 2:n // 2 + 16384] *= 1e-30
    flat[n // 3:n // 3 + 64] = 0.0125
    return W


@pytest.mark.parametrize("fmt", sorted(FMTS))
@pytest.mark.parametrize("shape", [(256, 1024), (3, 16384 + 64 * 5 + 7), (1032, 4160), (4096, 4096)])
def test_quantize_dequantize_bit_exact(lib, fmt, shape):
    W = _awkward_weight(*shape, seed=70 + shape[0])
    w, oq = _signed(W, fmt)
    got = q.dequantize(w).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, onf4.dequantize_nf4(oq))


def test_single_block_and_constant_tensor(lib):
    for W in (torch.full((1, 40), 0.5), torch.full((64, 256), 0.03), torch.zeros(8, 64)):
        _signed(W.float().contiguous())


def test_mean_does_not_depend_on_block_order(lib):
    W = qi.make_weight(512, 4096, seed=80)
    w0, _ = _signed(W)
    g = torch.Generator().manual_seed(81)
    perm = torch.randperm(W.numel() // 16384, generator=g)
    Wp = W.view(-1, 16384)[perm].reshape(W.shape).contiguous()     # the same blocks, groups reordered
    w1 = q.quantize_nf4(Wp.cuda(), dq=q.DQ_SIGNED)
    torch.cuda.synchronize()
    assert torch.equal(w0.offset.view(torch.int32), w1.offset.view(torch.int32))
    inv = torch.argsort(perm).cuda()
    assert torch.equal(w1.absmax_q.view(-1, 256)[inv].reshape(-1), w0.absmax_q)


@pytest.mark.parametrize("M,N,K,r", [(1, 776, 2112, 24), (4, 4096, 4096, 64), (12, 520, 704, 16),
                                     (96, 512, 448, 64), (300, 1032, 1152, 32), (1024, 1024, 2048, 64)])
def test_linear_parity(lib, M, N, K, r):
    case = qi.LinearCase(f"dqs_{M}_{N}_{K}_{r}", M, N, K, r, 16.0, 700 + M + N + K + r)
    d = qi.make_linear(case)
    w, oq = _signed(d["W"])
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


def test_signed_constants_error_on_the_gpu(lib):
    """The ablation through the library: the signed constants are closer to the
    exact block absmax than the plain ones on Gaussian weights, and the weight
    reconstruction error is the oracle's for both readings."""
    W = qi.make_weight(1024, 4096, seed=82)
    W64 = W.numpy().astype(np.float64)
    err = {}
    for name, dq in (("plain", q.DQ_PLAIN), ("signed", q.DQ_SIGNED)):
        w = q.quantize_nf4(W.cuda(), dq=dq)
        Wd = q.dequantize(w).float().cpu().numpy().astype(np.float64)
        err[name] = float(np.linalg.norm(Wd - W64) / np.linalg.norm(W64))
        assert err[name] == pytest.approx(onf4.reconstruction_error(W.numpy(), "nf4", name), rel=1e-12)
    assert abs(err["signed"] - err["plain"]) <= 0.01 * err["plain"], err
