"""Few-token forward (M <= 16, the dequant-GEMV kernels) against the fp64 oracle.

Covers one and two token tiles (M <= 8, M > 8), ragged N (N % 16 == 8), K not
a multiple of the 256-wide step, adapter ranks that are not multiples of 16,
tiles finished by one warp and tiles split over several warps (fixed-order
reduction), the LLaMA-7B projections at the decode token counts, and
run-to-run determinism."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from tests.gpu_util import TOL, assert_weight_bits, f64, gpu_weight, oracle_weight, rel

pytestmark = pytest.mark.gpu


def _fwd_case(case: qi.LinearCase, M: int | None = None, check_bits: bool = True):
    d = qi.make_linear(case, with_dy=False, M=M)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    if check_bits:
        assert_weight_bits(w, oq)
    X, A, B = d["X"].cuda(), d["A"].cuda(), d["B"].cuda()
    Y, H = q.linear_fwd(w, X, A, B, d["s"])
    Y2, H2 = q.linear_fwd(w, X, A, B, d["s"])
    torch.cuda.synchronize()
    assert q.device_status() == 0
    Yr, Hr = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    errs = {"Y": rel(f64(Y), Yr), "H": rel(f64(H), Hr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)
    # fixed reduction order: identical bits on a second call
    assert torch.equal(Y.view(torch.int16), Y2.view(torch.int16))
    assert torch.equal(H.view(torch.int32), H2.view(torch.int32))
    return errs


@pytest.mark.parametrize("M", [1, 2, 7, 8, 9, 15, 16])
def test_token_counts_ragged(lib, M):
    # N % 16 == 8, K = 2112 (8.25 steps of 256), r = 24: split tiles and a partial adapter step
    _fwd_case(qi.LinearCase(f"gemv_{M}", M, 776, 2112, 24, 16.0, 200 + M))


@pytest.mark.parametrize("N,K,r", [
    (8, 64, 8),          # one half-empty tile, one block column
    (256, 256, 8),       # every tile owned by one warp
    (392, 640, 40),      # r % 16 == 8
    (1032, 1152, 256),   # largest rank
    (2048, 4160, 64),    # many split tiles, K % 256 == 64
])
def test_shapes(lib, N, K, r):
    for M in (1, 12):
        _fwd_case(qi.LinearCase(f"gemv_shape_{N}_{K}_{r}_{M}", M, N, K, r, 16.0, 300 + N + K + r + M))


@pytest.mark.parametrize("case", qi.LLAMA7B, ids=lambda c: c.name)
def test_llama7b_decode_tokens(lib, case):
    """The decode shapes the bench times: the LLaMA-7B projections at 1, 4
    and 16 tokens, Y and H in full against the oracle."""
    d = qi.make_linear(case, with_dy=False, M=16)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    assert_weight_bits(w, oq)
    A, B = d["A"].cuda(), d["B"].cuda()
    A64, B64 = f64(d["A"]), f64(d["B"])
    for M in qi.GEMV_TOKENS:
        X = d["X"][:M].contiguous()
        Y, H = q.linear_fwd(w, X.cuda(), A, B, d["s"])
        torch.cuda.synchronize()
        assert q.device_status() == 0
        Yr, Hr = olin.lora_linear_fwd(Wd, f64(X), A64, B64, d["s"])
        errs = {"Y": rel(f64(Y), Yr), "H": rel(f64(H), Hr)}
        for k, e in errs.items():
            assert e <= TOL, (M, k, errs)


def test_gemv_matches_tensor_core_path(lib):
    """The same rows through both forward paths: 16 tokens alone (GEMV) and
    as the first 16 rows of a 17-token call (tensor-core GEMM) agree to the
    parity tolerance."""
    case = qi.LinearCase("gemv_vs_tc", 17, 1040, 1536, 32, 16.0, 77)
    d = qi.make_linear(case, with_dy=False)
    w = gpu_weight(d["W"])
    X, A, B = d["X"].cuda(), d["A"].cuda(), d["B"].cuda()
    Y17, _ = q.linear_fwd(w, X, A, B, d["s"])
    Y16, _ = q.linear_fwd(w, X[:16].contiguous(), A, B, d["s"])
    torch.cuda.synchronize()
    assert rel(f64(Y16), f64(Y17[:16])) <= TOL


@pytest.mark.parametrize("M", [1, 16])
def test_any_workspace_contents(lib, M):
    """The grid barrier's word lives in the caller's workspace and is tagged per
    launch: whatever an unused workspace holds (random bytes, all ones, zeros),
    the result is the same bits, call after call."""
    case = qi.LinearCase(f"ws_{M}", M, 1032, 2112, 24, 16.0, 61 + M)
    d = qi.make_linear(case, with_dy=False)
    w = q.quantize_nf4(d["W"].cuda())
    X, A, B = d["X"].cuda(), d["A"].cuda(), d["B"].cuda()
    need = q.workspace_bytes(q.QLORA_OP_FWD, M, case.N, case.K, case.r)
    g = torch.Generator(device="cpu").manual_seed(5)
    fills = [torch.randint(0, 256, (need,), dtype=torch.uint8, generator=g).cuda(),
             torch.full((need,), 255, dtype=torch.uint8, device="cuda"),
             torch.zeros(need, dtype=torch.uint8, device="cuda")]
    outs = []
    for ws in fills:
        for _ in range(2):
            Y, _ = q.linear_fwd(w, X, A, B, case.s, save_h=False, workspace=ws)
            outs.append(Y.clone())
    torch.cuda.synchronize()
    assert q.device_status() == 0
    for Y in outs[1:]:
        assert torch.equal(Y, outs[0])
