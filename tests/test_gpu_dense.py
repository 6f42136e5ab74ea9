"""The linear on a base weight from any quantizer ("ModuLoRA", abstract: the
low-precision weights of a black-box quantization module are materialized
in each pass):

- with W' = the library's own dequantized NF4 weight, the dense calls equal
  the packed calls bit for bit wherever those take the pair kernel (M > 128);
- with a weight from another quantizer (8-bit rows, dequantized by torch),
  forward and backward against the fp64 oracle, including token counts the
  packed path would route to the few-token kernel;
- the materializing call runs the caller's dequantizer and equals the dense
  call bit for bit.
"""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from tests.gpu_util import TOL, f64, rel

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,r", [(300, 1032, 1152, 32), (1024, 1024, 2048, 64), (4096, 4096, 4096, 64)])
def test_dense_equals_packed(lib, M, N, K, r):
    case = qi.LinearCase(f"dense_{M}_{N}_{K}", M, N, K, r, 16.0, 800 + M + N + K)
    d = qi.make_linear(case)
    w = q.quantize_nf4(d["W"].cuda())
    Wd = q.dequantize(w)
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y1, H1 = q.linear_fwd(w, X, A, B, d["s"])
    Y2, H2 = q.linear_fwd_dense(Wd, X, A, B, d["s"])
    g1 = q.linear_bwd(w, X, dY, A, B, d["s"], H=H1)
    g2 = q.linear_bwd_dense(Wd, X, dY, A, B, d["s"], H=H2)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert torch.equal(Y1, Y2) and torch.equal(H1, H2)
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


def _int8_rows(W: torch.Tensor) -> torch.Tensor:
    """Another quantizer: symmetric 8-bit per output row, dequantized to bf16."""
    scale = W.abs().amax(dim=1, keepdim=True) / 127.0
    return (torch.round(W / scale).clamp(-127, 127) * scale).to(torch.bfloat16)


@pytest.mark.parametrize("M,N,K,r", [(1, 776, 2112, 24), (12, 520, 704, 16), (96, 512, 448, 64),
                                     (300, 1032, 1152, 32)])
def test_dense_from_another_quantizer(lib, M, N, K, r):
    case = qi.LinearCase(f"int8_{M}_{N}_{K}", M, N, K, r, 16.0, 900 + M + N + K)
    d = qi.make_linear(case)
    Wd = _int8_rows(d["W"].cuda())
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    Y, H = q.linear_fwd_dense(Wd, X, A, B, d["s"])
    dX, dA, dB = q.linear_bwd_dense(Wd, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    W64 = f64(Wd)
    Yr, Hr = olin.lora_linear_fwd(W64, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    dXr, dAr, dBr = olin.lora_linear_bwd(W64, f64(d["X"]), f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
    errs = {"Y": rel(f64(Y), Yr), "H": rel(f64(H), Hr), "dX": rel(f64(dX), dXr), "dA": rel(f64(dA), dAr),
            "dB": rel(f64(dB), dBr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)


def test_materialized_runs_the_callers_dequantizer(lib):
    M, N, K, r = 256, 1024, 1024, 32
    case = qi.LinearCase("materialized", M, N, K, r, 16.0, 950)
    d = qi.make_linear(case)
    Wc = d["W"].cuda()
    X, A, B = (d[k].cuda() for k in ("X", "A", "B"))
    calls = []

    def materialize(out):
        calls.append(out.shape)
        out.copy_(_int8_rows(Wc))
    Y1, H1 = q.linear_fwd_materialized(materialize, N, K, X, A, B, d["s"])
    Y2, H2 = q.linear_fwd_dense(_int8_rows(Wc), X, A, B, d["s"])
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert calls == [(N, K)]
    assert torch.equal(Y1, Y2) and torch.equal(H1, H2)
