"""The LLaMA-65B-shaped projections (8192 tokens, r = 64) in the launch
configuration the kernels use at that size, against the oracle.

- 8192 x 8192: weight bit-exact in full; Y and dX on sampled token rows,
  dA and dB in full.
- 22016 x 8192: codes, 8-bit constants, group scales and the dequantized
  weight bit-exact on row slabs aligned to whole double-quantization groups
  (two rows per group at K = 8192); Y and dB on those rows."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from oracle import nf4 as onf4
from tests.gpu_util import TOL, assert_weight_bits, f64, gpu_weight, oracle_weight, rel

pytestmark = pytest.mark.gpu


def _chunked_grads(X, dY, A, B, s, rows=1024):
    """dA, dB from the oracle's adapter gradients, summed over token chunks in fp64."""
    dA = np.zeros(A.shape, np.float64)
    dB = np.zeros(B.shape, np.float64)
    for m0 in range(0, X.shape[0], rows):
        a, b = olin.lora_adapter_grads(X[m0:m0 + rows].astype(np.float64), dY[m0:m0 + rows].astype(np.float64),
                                       A, B, s)
        dA += a
        dB += b
    return dA, dB


def test_llama65b_square_projection(lib):
    case = qi.LLAMA65B[0]
    d = qi.make_linear(case)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    assert_weight_bits(w, oq)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd(w, X, A, B, d["s"])
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    rows = np.sort(np.random.default_rng(case.seed).choice(case.M, 32, replace=False))
    A64, B64 = f64(d["A"]), f64(d["B"])
    Yr, _ = olin.lora_linear_fwd(Wd, f64(d["X"][rows]), A64, B64, d["s"])
    dXr = olin.lora_input_grad(Wd, f64(d["dY"][rows]), A64, B64, d["s"])
    dAr, dBr = _chunked_grads(d["X"].float().numpy(), d["dY"].float().numpy(), A64, B64, d["s"])
    errs = {"Y": rel(f64(Y[rows]), Yr), "dX": rel(f64(dX[rows]), dXr), "dA": rel(f64(dA), dAr),
            "dB": rel(f64(dB), dBr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)


def test_llama65b_wide_weight_slabs(lib):
    case = qi.LLAMA65B[1]            # 22016 x 8192
    d = qi.make_linear(case)
    w = gpu_weight(d["W"])
    Wdev = q.dequantize(w)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd(w, X, A, B, d["s"])
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    K = case.K
    per_group_rows = 16384 // K      # 2
    A64 = f64(d["A"])
    tokens = np.sort(np.random.default_rng(case.seed).choice(case.M, 16, replace=False))
    for r0 in (0, 10000, case.N - 64):
        r0 -= r0 % per_group_rows
        rows = slice(r0, r0 + 64)
        oq = onf4.quantize_nf4(d["W"][rows].numpy())
        g0 = r0 * K // 16384
        assert np.array_equal(w.codes[r0 * K // 2:(r0 + 64) * K // 2].cpu().numpy(), oq["codes"])
        assert np.array_equal(w.absmax_q[r0 * K // 64:(r0 + 64) * K // 64].cpu().numpy(), oq["absmax_q"])
        assert np.array_equal(w.group_scale[g0:g0 + 64 // per_group_rows].cpu().numpy().view(np.uint32),
                              oq["group_scale"].view(np.uint32))
        got = Wdev[rows].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, onf4.dequantize_nf4(oq))
        Wd = onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64)
        B_rows = f64(d["B"][rows])
        Yr, _ = olin.lora_linear_fwd(Wd, f64(d["X"][tokens]), A64, B_rows, d["s"])   # Y columns = these rows
        assert rel(f64(Y[tokens][:, rows]), Yr) <= TOL
        _, dBr = _chunked_grads(d["X"].float().numpy(), d["dY"][:, rows].float().numpy(), A64, B_rows, d["s"])
        assert rel(f64(dB[rows]), dBr) <= TOL
