"""The low-rank plus quantized decomposition ("LQ-LoRA: Low-rank Plus
Quantized Matrix Decomposition for Efficient Language Model Finetuning",
abstract) through the library, against the oracle:

- the residual quantization step bit-exact (codes, 8-bit constants, scales)
  for given fp32 factors, both block-constant readings;
- the rank-r step against the oracle's randomized SVD with the same test
  matrix (product L1 L2, relative Frobenius), with and without a quantized
  part, and near the Eckart-Young optimum;
- the whole alternation: error history close to the oracle's, each rank-r
  step never worse than the factors it replaces, far below plain NF4, and
  bit-identical on a second run;
- the LLaMA-7B q-projection shape (4096 x 4096, r = 64, l = 72) at full size.
"""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import lq, nf4 as onf4

pytestmark = pytest.mark.gpu

PRODUCT_TOL = 1e-4    # L1 L2 of the fp32 GPU path vs the fp64 oracle with the same test matrix


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.parametrize("dq", ["plain", "signed"])
@pytest.mark.parametrize("shape,r", [((256, 512), 16), ((300, 1000), 8), ((1024, 2048), 64)])
def test_quantize_residual_bit_exact(lib, shape, r, dq):
    N, K = shape
    W = qi.make_lowrank_weight(N, K, r, seed=90 + N)
    L1o, L2o, _ = lq.truncated_svd(W.numpy(), r)
    L1, L2 = L1o.astype(np.float32), L2o.astype(np.float32)
    E = lq.lowrank_residual(W.numpy(), L1, L2)
    oq = onf4.quantize_nf4(E, dq=dq)
    w = q.lq_quantize_residual(W.cuda(), torch.from_numpy(L1).cuda(), torch.from_numpy(L2).cuda(),
                               dq=q.DQ_SIGNED if dq == "signed" else q.DQ_PLAIN)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert np.array_equal(w.codes.cpu().numpy(), oq["codes"])
    assert np.array_equal(w.absmax_q.cpu().numpy(), oq["absmax_q"])
    assert np.array_equal(w.scales.cpu().numpy().view(np.uint32), oq["group_scale"].view(np.uint32))


@pytest.mark.parametrize("with_q", [False, True])
@pytest.mark.parametrize("shape,r,l,power", [((256, 512), 16, 24, 2), ((512, 384), 32, 40, 1), ((1024, 2048), 64, 72, 2)])
def test_lowrank_step_matches_the_oracle(lib, shape, r, l, power, with_q):
    N, K = shape
    W = qi.make_lowrank_weight(N, K, r, seed=95 + N)
    Om = qi.make_test_matrix(K, l, seed=96 + K)
    Wd = W.cuda()
    Q = q.quantize_nf4(Wd) if with_q else None
    L1, L2 = q.lq_lowrank(Wd, Q, Om.cuda(), r, power)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    if with_q:
        R = lq.quant_residual(W.numpy(), onf4.dequantize_nf4(onf4.quantize_nf4(W.numpy())))
    else:
        R = W.numpy()
    a, b, _ = lq.randomized_svd(R, Om.numpy(), r, power)
    P = L1.double().cpu().numpy() @ L2.double().cpu().numpy()
    assert _rel(P, a @ b) <= PRODUCT_TOL
    e, f, _ = lq.truncated_svd(R, r)
    R64 = R.astype(np.float64)
    assert np.linalg.norm(R64 - P) <= 1.05 * np.linalg.norm(R64 - e @ f)


def test_decomposition_matches_the_oracle_and_repeats(lib):
    N, K, r, l, power, iters = 512, 1024, 32, 40, 2, 3
    W = qi.make_lowrank_weight(N, K, r, seed=97)
    Om = qi.make_test_matrix(K, l, seed=98)
    ref = lq.lq_decompose(W.numpy(), r, iters, Omega=Om.numpy(), power=power)
    runs = []
    for _ in range(2):
        w, L1, L2, err = q.lq_decompose(W.cuda(), r, Om.cuda(), power=power, iters=iters)
        torch.cuda.synchronize()
        assert q.device_status() == 0
        runs.append((w, L1, L2, err.cpu().numpy()))
    w, L1, L2, err = runs[0]
    assert torch.equal(runs[1][0].codes, w.codes) and torch.equal(runs[1][1], L1) and torch.equal(runs[1][2], L2)
    assert np.array_equal(runs[1][3], err)
    pre, post = err[:, 0], err[:, 1]
    assert np.all(post <= pre * (1 + 1e-6))
    assert post[-1] < 0.6 * ref["plain_err"]
    np.testing.assert_allclose(pre, ref["pre"], rtol=2e-3)
    np.testing.assert_allclose(post, ref["err"], rtol=2e-3)
    # the reported error is the error of the returned parts
    e = lq.decomposition_error(W.numpy(), q.dequantize(w).view(torch.int16).cpu().numpy().view(np.uint16),
                               L1.cpu().numpy(), L2.cpu().numpy())
    assert e == pytest.approx(post[-1], rel=1e-9)
    # the quantized parts differ only where a code sits on a threshold for inputs a rounding apart
    codes_o = onf4.unpack_nibbles(ref["q"]["codes"], N * K)
    codes_g = onf4.unpack_nibbles(w.codes.cpu().numpy(), N * K)
    assert np.mean(codes_o != codes_g) <= 1e-3


def test_llama7b_projection_shape(lib):
    N = K = 4096
    r, l = 64, 72
    W = qi.make_lowrank_weight(N, K, r, seed=99)
    Om = qi.make_test_matrix(K, l, seed=100)
    plain = q.quantize_nf4(W.cuda())
    Wd = q.dequantize(plain).double()
    plain_err = float((Wd - W.cuda().double()).norm() / W.cuda().double().norm())
    w, L1, L2, err = q.lq_decompose(W.cuda(), r, Om.cuda(), power=2, iters=2)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    e = err.cpu().numpy()
    assert np.isfinite(e).all() and np.all(e[:, 1] <= e[:, 0] * (1 + 1e-6))
    # at this size the planted part holds about 30 % of the energy (57 % at 256 x 512), so the
    # gain over plain NF4 is smaller: measured 0.0712 against 0.0920 after two rounds
    assert e[-1, 1] < 0.85 * plain_err and e[-1, 1] <= e[0, 1], (e, plain_err)
    Wq = q.dequantize(w).double()
    direct = float((W.cuda().double() - Wq - L1.double() @ L2.double()).norm() / W.cuda().double().norm())
    assert direct == pytest.approx(e[-1, 1], rel=1e-6)
