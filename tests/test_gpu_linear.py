"""GPU parity of the QLoRA linear (forward and backward) against the fp64
oracle: relative Frobenius error <= 2e-3 on Y, dX, dA and dB."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from tests.gpu_util import TOL, assert_weight_bits, f64, gpu_weight, oracle_weight, rel

pytestmark = pytest.mark.gpu


def _run_case(case: qi.LinearCase, M: int | None = None, save_h: bool = True):
    d = qi.make_linear(case, M=M)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    assert_weight_bits(w, oq)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd(w, X, A, B, d["s"], save_h=save_h)
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    Yr, Hr = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    dXr, dAr, dBr = olin.lora_linear_bwd(Wd, f64(d["X"]), f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
    errs = {"Y": rel(f64(Y), Yr), "dX": rel(f64(dX), dXr), "dA": rel(f64(dA), dAr), "dB": rel(f64(dB), dBr)}
    if H is not None:
        errs["H"] = rel(f64(H), Hr)
    for k, e in errs.items():
        assert e <= TOL, (k, errs)
    return errs


def test_small_config(lib):
    _run_case(qi.SMALL)


@pytest.mark.parametrize("M,N,K,r", [
    (300, 520, 704, 24),      # ragged in every tiled dimension, one partial adapter step
    (128, 256, 256, 64),      # exactly one tile
    (257, 264, 1088, 72),     # two adapter steps, the second partial
    (96, 512, 448, 128),
    (200, 128, 640, 256),
    (64, 8, 64, 8),           # minimal shapes
    (129, 392, 640, 64),      # first size on the CTA-pair kernel (one pair, odd CTA mostly empty)
    (256, 512, 1024, 32),     # exactly one pair tile
    (520, 1800, 1344, 16),    # several pairs, ragged N and K (K % 128 != 0)
])
def test_ragged_shapes(lib, M, N, K, r):
    _run_case(qi.LinearCase(f"ragged_{M}_{N}_{K}_{r}", M, N, K, r, 16.0, 100 + M + N + K + r))


def test_recompute_h_when_not_saved(lib):
    _run_case(qi.LinearCase("nosave", 192, 320, 512, 16, 32.0, 17), save_h=False)


@pytest.mark.parametrize("M", [1, 4, 16, 17])
def test_few_tokens(lib, M):
    _run_case(qi.LinearCase(f"few_{M}", M, 512, 1024, 64, 16.0, 40 + M))


def test_adapter_only_special_case(lib):
    """A = 0: the forward is the plain dequantized GEMM and dA/dB vanish or
    reduce to closed forms (dA = s (dY B)^T X needs B; with A = 0, dB = 0)."""
    case = qi.LinearCase("a_zero", 256, 512, 512, 16, 16.0, 21)
    d = qi.make_linear(case)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    X, B, dY = d["X"].cuda(), d["B"].cuda(), d["dY"].cuda()
    A = torch.zeros_like(d["A"]).cuda()
    Y, H = q.linear_fwd(w, X, A, B, case.s)
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, case.s, H=H)
    torch.cuda.synchronize()
    Yr = f64(d["X"]) @ Wd.T
    assert rel(f64(Y), Yr) <= TOL
    assert torch.count_nonzero(dB).item() == 0
    assert rel(f64(dX), f64(d["dY"]) @ Wd) <= TOL


@pytest.mark.parametrize("case", qi.LLAMA7B, ids=lambda c: c.name)
def test_llama7b_projection_sampled(lib, case):
    """Full-size projection (M = 4096, r = 64) in the launch configuration the
    bench times; Y and dX checked on 48 sampled token rows against the oracle,
    dA and dB in full."""
    d = qi.make_linear(case)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    assert_weight_bits(w, oq)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd(w, X, A, B, d["s"])
    dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    rows = np.random.default_rng(case.seed).choice(case.M, 48, replace=False)
    rows.sort()
    A64, B64 = f64(d["A"]), f64(d["B"])
    Yr, _ = olin.lora_linear_fwd(Wd, f64(d["X"][rows]), A64, B64, d["s"])
    dXr = olin.lora_input_grad(Wd, f64(d["dY"][rows]), A64, B64, d["s"])
    dAr, dBr = olin.lora_adapter_grads(f64(d["X"]), f64(d["dY"]), A64, B64, d["s"])
    errs = {"Y": rel(f64(Y[rows]), Yr), "dX": rel(f64(dX[rows]), dXr), "dA": rel(f64(dA), dAr),
            "dB": rel(f64(dB), dBr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)
