"""Pins of the oracle's low-rank plus quantized decomposition ("LQ-LoRA:
Low-rank Plus Quantized Matrix Decomposition for Efficient Language Model
Finetuning", abstract): the fp64 low-rank residual element by element, the
truncated SVD against the Eckart-Young optimum computed another way, the
randomized SVD against exact cases, and the alternation against the
guarantee of its first round."""

import numpy as np
import pytest

import qlora_inputs as qi
from oracle import lq, nf4


def test_lowrank_product_matches_a_scalar_loop():
    rng = np.random.default_rng(40)
    L1 = rng.standard_normal((3, 4)).astype(np.float32)
    L2 = rng.standard_normal((4, 5)).astype(np.float32)
    W = rng.standard_normal((3, 5)).astype(np.float32)
    P = lq.lowrank_product(L1, L2)
    E = lq.lowrank_residual(W, L1, L2)
    for n in range(3):
        for k in range(5):
            p = 0.0
            for j in range(4):
                p = p + float(L1[n, j]) * float(L2[j, k])     # Python floats: fp64, products exact
            assert P[n, k] == p
            assert E[n, k] == np.float32(float(W[n, k]) - p)
    assert np.array_equal(lq.lowrank_residual(W, np.zeros((3, 4)), np.zeros((4, 5))), W)


def test_lowrank_residual_rounds_once_from_fp64():
    # 1 + 2^-30 survives in fp64 but not fp32: the subtraction is done before the fp32 rounding
    W = np.array([[1.0]], np.float32)
    L1 = np.array([[2.0 ** -15]], np.float32)
    L2 = np.array([[-(2.0 ** -15)]], np.float32)
    assert lq.lowrank_product(L1, L2)[0, 0] == -(2.0 ** -30)
    assert lq.lowrank_residual(W, L1, L2)[0, 0] == np.float32(1.0)
    L2b = np.array([[-(2.0 ** -9)]], np.float32)          # 1 + 2^-24: a tie, rounds to even (1.0)
    assert lq.lowrank_residual(W, L1, L2b)[0, 0] == np.float32(1.0)
    L2c = np.array([[-(3 * 2.0 ** -10)]], np.float32)     # 1 + 1.5 * 2^-24 rounds up
    assert lq.lowrank_residual(W, L1, L2c)[0, 0] == np.float32(1.0 + 2.0 ** -23)


def test_quant_residual_of_a_representable_weight_is_zero():
    W = nf4.bf16_bits_to_f32(nf4.bf16_rne_bits(np.random.default_rng(41).standard_normal(256).astype(np.float32)))
    assert np.all(lq.quant_residual(W.reshape(4, 64), nf4.bf16_rne_bits(W)) == 0)


def test_truncated_svd_is_the_eckart_young_optimum():
    rng = np.random.default_rng(42)
    R = rng.standard_normal((60, 90))
    r = 7
    L1, L2, _ = lq.truncated_svd(R, r)
    lam = np.sort(np.linalg.eigvalsh(R @ R.T))[::-1]          # another route to the singular values
    assert np.linalg.norm(R - L1 @ L2) ** 2 == pytest.approx(lam[r:].sum(), rel=1e-10)
    assert np.allclose(L1.T @ L1, np.diag(np.sqrt(lam[:r])), atol=1e-10)
    assert np.allclose(L2 @ L2.T, np.diag(np.sqrt(lam[:r])), atol=1e-10)
    low = rng.standard_normal((60, 5)) @ rng.standard_normal((5, 90))
    a, b, _ = lq.truncated_svd(low, r)
    assert np.linalg.norm(a @ b - low) <= 1e-12 * np.linalg.norm(low)


def test_randomized_svd_exact_and_gapped_cases():
    rng = np.random.default_rng(43)
    N, K, r, l = 120, 200, 8, 16
    Om = rng.standard_normal((K, l))
    low = rng.standard_normal((N, 6)) @ rng.standard_normal((6, K))       # rank 6 <= r: captured exactly
    a, b, _ = lq.randomized_svd(low, Om, r, 0)
    assert np.linalg.norm(a @ b - low) <= 1e-10 * np.linalg.norm(low)
    U, _ = np.linalg.qr(rng.standard_normal((N, N)))
    V, _ = np.linalg.qr(rng.standard_normal((K, N)))
    s = np.concatenate([np.linspace(20, 10, r), np.linspace(0.5, 0.1, N - r)])    # gap of 20 at r
    R = (U * s) @ V.T
    e, f, _ = lq.truncated_svd(R, r)
    # subspace iteration shrinks the unwanted directions by (s_{r+1} / s_r)^(2 power + 1) = 0.05^5
    # per round relative to the wanted ones: about 1e-7 of the product for power = 2, 1e-10 for 3
    diff = []
    for power in (2, 3):
        a, b, sr = lq.randomized_svd(R, Om, r, power)
        diff.append(np.linalg.norm(a @ b - e @ f) / np.linalg.norm(e @ f))
    assert diff[0] <= 1e-6 and diff[1] <= 1e-8, diff
    assert np.allclose(sr, s[:r], rtol=1e-10)
    assert np.allclose(a.T @ a, np.diag(sr), atol=1e-9) and np.allclose(b @ b.T, np.diag(sr), atol=1e-9)
    z1, z2, zs = lq.randomized_svd(np.zeros((N, K)), Om, r, 1)
    assert not z1.any() and not z2.any() and not zs.any()


def test_randomized_svd_near_optimal_on_a_flat_spectrum():
    rng = np.random.default_rng(44)
    R = rng.standard_normal((256, 512))
    r = 16
    e, f, _ = lq.truncated_svd(R, r)
    opt = np.linalg.norm(R - e @ f)
    ratios = []
    for power in (0, 2):
        a, b, _ = lq.randomized_svd(R, rng.standard_normal((512, r + 8)), r, power)
        ratios.append(np.linalg.norm(R - a @ b) / opt)
    assert 1.0 <= ratios[1] <= 1.03 and ratios[1] < ratios[0], ratios


def test_alternation_guarantees_and_the_planted_part():
    N, K, r = 256, 512, 16
    W = qi.make_lowrank_weight(N, K, r, seed=45).numpy()
    rng = np.random.default_rng(45)                       # the planted part: W minus its Gaussian draw
    planted = W.astype(np.float64) - rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    out = lq.lq_decompose(W, r, 4)
    # each SVD step is the best rank-r fit of the current residual: never worse than keeping L
    for p, e in zip(out["pre"], out["err"]):
        assert e <= p
    # the principal part of W leaves a near-Gaussian remainder, which NF4 stores far better
    assert out["err"][-1] < 0.6 * out["plain_err"]
    assert out["err"][-1] <= out["err"][0]
    L = lq.lowrank_product(out["L1"], out["L2"])
    assert np.linalg.norm(L - planted) <= 0.35 * np.linalg.norm(planted)
    q = out["q"]
    assert lq.decomposition_error(W, nf4.dequantize_nf4(q), out["L1"], out["L2"]) == pytest.approx(out["err"][-1])
    Om = qi.make_test_matrix(K, r + 8, seed=46).numpy()
    outr = lq.lq_decompose(W, r, 4, Omega=Om, power=2)
    assert outr["err"][-1] <= out["err"][-1] * 1.02
