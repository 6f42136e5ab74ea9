"""Pins for the fp64 LoRA linear oracle (CPU only).

The backward is pinned against the forward by finite differences and adjoint
identities; the forward by the LoRA merge identity and by the adapter-free
special case, both through torch's dense linear (an independent routine).
"""

import numpy as np
import torch

from oracle import linear


def _case(rng, M=5, N=7, K=6, r=3):
    return (rng.standard_normal((N, K)), rng.standard_normal((M, K)), rng.standard_normal((r, K)),
            rng.standard_normal((N, r)), rng.standard_normal((M, N)))


def test_fwd_merge_identity():
    rng = np.random.default_rng(0)
    W, X, A, B, _ = _case(rng)
    s = 0.75
    Y, H = linear.lora_linear_fwd(W, X, A, B, s)
    merged = torch.from_numpy(W) + s * torch.from_numpy(B) @ torch.from_numpy(A)
    ref = torch.nn.functional.linear(torch.from_numpy(X), merged).numpy()
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(H, torch.nn.functional.linear(torch.from_numpy(X), torch.from_numpy(A)).numpy())


def test_fwd_without_adapter_is_dense_linear():
    rng = np.random.default_rng(1)
    W, X, A, B, dY = _case(rng)
    for A_, B_ in ((np.zeros_like(A), B), (A, np.zeros_like(B))):
        Y, _ = linear.lora_linear_fwd(W, X, A_, B_, 2.0)
        ref = torch.nn.functional.linear(torch.from_numpy(X), torch.from_numpy(W)).numpy()
        assert np.allclose(Y, ref, rtol=1e-13, atol=1e-13)
    dX, dA, dB = linear.lora_linear_bwd(W, X, dY, A, np.zeros_like(B), 2.0)
    assert np.all(dA == 0)
    assert np.allclose(dX, (torch.from_numpy(dY) @ torch.from_numpy(W)).numpy())
    _, _, dB0 = linear.lora_linear_bwd(W, X, dY, np.zeros_like(A), B, 2.0)
    assert np.all(dB0 == 0)


def test_bwd_finite_differences():
    """dX, dA, dB equal the derivatives of L = sum(dY * Y) taken numerically
    from the forward (L is linear in X and in each adapter separately, so a
    central difference is exact up to rounding)."""
    rng = np.random.default_rng(2)
    W, X, A, B, dY = _case(rng, M=4, N=5, K=6, r=2)
    s = 1.5

    def L(X_, A_, B_):
        return float(np.sum(dY * linear.lora_linear_fwd(W, X_, A_, B_, s)[0]))

    dX, dA, dB = linear.lora_linear_bwd(W, X, dY, A, B, s)
    h = 1e-3
    for name, base, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        num = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            p, m = base.copy(), base.copy()
            p[idx] += h
            m[idx] -= h
            args = {"X": X, "A": A, "B": B}
            args[name] = p
            lp = L(args["X"], args["A"], args["B"])
            args[name] = m
            lm = L(args["X"], args["A"], args["B"])
            num[idx] = (lp - lm) / (2 * h)
        assert np.allclose(grad, num, rtol=1e-7, atol=1e-8), name


def test_adjoint_identities():
    rng = np.random.default_rng(3)
    W, X, A, B, dY = _case(rng, M=9, N=11, K=13, r=4)
    s = 0.25
    Y, _ = linear.lora_linear_fwd(W, X, A, B, s)
    Yb, _ = linear.lora_linear_fwd(W, X, np.zeros_like(A), B, s)
    dX, dA, dB = linear.lora_linear_bwd(W, X, dY, A, B, s)
    # Y is linear in X:        <dY, Y> = <dX, X>
    assert np.isclose(np.sum(dY * Y), np.sum(dX * X), rtol=1e-12)
    # the LoRA term is linear in A and in B:  <dY, Y - Y_base> = <dA, A> = <dB, B>
    lora = np.sum(dY * (Y - Yb))
    assert np.isclose(lora, np.sum(dA * A), rtol=1e-12)
    assert np.isclose(lora, np.sum(dB * B), rtol=1e-12)


def test_rel_frobenius():
    a = np.ones((3, 3))
    assert linear.rel_frobenius(a, a) == 0.0
    assert np.isclose(linear.rel_frobenius(a * 1.001, a), 1e-3)
    assert linear.rel_frobenius(np.zeros(2), np.zeros(2)) == 0.0
