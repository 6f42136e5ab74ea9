"""Oracle: low-rank plus quantized decomposition of a frozen weight (CPU).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  numpy, fp64 unless a step
fixes fp32; the truncated SVD is numpy's (LAPACK) in fp64.

Source: "LQ-LoRA: Low-rank Plus Quantized Matrix Decomposition for Efficient
Language Model Finetuning", abstract.  Each pretrained matrix is split, by an
iterative algorithm, into a high-precision low-rank part and a quantized
part; finetuning keeps the quantized part fixed and trains the low-rank one.
The abstract gives no equations.  Reading (the plainest alternation the text
supports): the high-precision low-rank part starts as the principal rank-r
part of W itself, L1 L2 = best rank-r approximation of W, then each round t

    E_t        = W - L1 L2                     (what the quantized part must hold)
    Q_t        = quantize(E_t)                 (this library's 4-bit storage)
    pre_t      = ||W - dequant(Q_t) - L1 L2||_F / ||W||_F
    R_t        = W - dequant(Q_t)              (what the low-rank part must hold)
    L1, L2     = best rank-r approximation of R_t (truncated SVD),
                 L1 = U_r diag(sqrt(s_r)),  L2 = diag(sqrt(s_r)) V_r^T
    err_t      = ||W - dequant(Q_t) - L1 L2||_F / ||W||_F  (<= pre_t, Eckart-Young)

The precision of each step is fixed so that the quantizer sees the same fp32
input on both sides:
    E = fl32( fl64(W) - P ),  P = sum over j = 0 .. r-1 in that order of
        fl64(L1[n, j] * L2[j, k])  (fp64 running sum; each product of two fp32
        values is exact in fp64);
    R = fl32(W - W')          (W' the bf16 dequantized weight, an fp32 subtraction).
The ILP that picks bit-widths per matrix under a memory budget (the same
abstract) needs data statistics and is not part of this reading.
"""

from __future__ import annotations

import numpy as np

from . import nf4


def lowrank_product(L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """P = L1 L2 in fp64, accumulated over the rank index in order 0 .. r-1."""
    L1 = np.asarray(L1, np.float32).astype(np.float64)
    L2 = np.asarray(L2, np.float32).astype(np.float64)
    P = np.zeros((L1.shape[0], L2.shape[1]), np.float64)
    for j in range(L1.shape[1]):
        P += L1[:, j:j + 1] * L2[j:j + 1, :]
    return P


def lowrank_residual(W: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """E = fl32(fl64(W) - P), the input of the quantized part."""
    W = np.asarray(W, np.float32)
    return (W.astype(np.float64) - lowrank_product(L1, L2)).astype(np.float32)


def quant_residual(W: np.ndarray, Wq_bits: np.ndarray) -> np.ndarray:
    """R = fl32(W - W') with W' given as bf16 bit patterns."""
    W = np.asarray(W, np.float32)
    Wq = nf4.bf16_bits_to_f32(Wq_bits).reshape(W.shape)
    return (W - Wq).astype(np.float32)


def truncated_svd(R: np.ndarray, r: int):
    """(L1 [N, r], L2 [r, K], s [min(N,K)]) fp64: the best rank-r approximation
    L1 L2 of R in the Frobenius norm (Eckart-Young), with the singular values
    split evenly between the factors."""
    U, s, Vt = np.linalg.svd(np.asarray(R, np.float64), full_matrices=False)
    h = np.sqrt(s[:r])
    return U[:, :r] * h[None, :], h[:, None] * Vt[:r], s


def _orth(Y: np.ndarray) -> np.ndarray:
    """An orthonormal basis of the columns of Y (library QR, fp64)."""
    Q, _ = np.linalg.qr(Y)
    return Q


def randomized_svd(R: np.ndarray, Omega: np.ndarray, r: int, power: int):
    """Rank-r approximation L1 L2 of R by randomized subspace iteration (the
    range finder of Halko, Martinsson and Tropp, "Finding structure with
    randomness", with `power` rounds of subspace iteration), fp64.

    With the Gaussian test matrix Omega [K, l], l >= r:
        Q = orth(R Omega);  `power` times: Q = orth(R orth(R^T Q))
        B = Q^T R [l, K];   B B^T = U diag(lam) U^T, lam descending
        s = sqrt(lam[:r]);  L1 = Q U_r diag(sqrt(s)),  L2 = diag(1/sqrt(s)) U_r^T B
    (so L2 = diag(sqrt(s)) V_r^T and L1 L2 = Q U_r U_r^T B).  A component with
    s_i <= 1e-12 s_0 (numerically absent) gets zero columns / rows."""
    R = np.asarray(R, np.float64)
    Q = _orth(R @ np.asarray(Omega, np.float64))
    for _ in range(power):
        Q = _orth(R @ _orth(R.T @ Q))
    B = Q.T @ R
    lam, U = np.linalg.eigh(B @ B.T)
    order = np.argsort(lam)[::-1][:r]
    lam, Ur = lam[order], U[:, order]
    s = np.sqrt(np.maximum(lam, 0.0))
    keep = s > 1e-12 * s[0] if s[0] > 0 else np.zeros_like(s, bool)
    h = np.where(keep, np.sqrt(s), 1.0)
    L1 = (Q @ Ur) * np.where(keep, h, 0.0)[None, :]
    L2 = (Ur.T @ B) * np.where(keep, 1.0 / h, 0.0)[:, None]
    return L1, L2, s


def lq_decompose(W: np.ndarray, r: int, iters: int, fmt: str = "nf4", dq: str = "plain",
                 Omega: np.ndarray | None = None, power: int = 2):
    """The alternation above for `iters` rounds.  Every rank-r step is the exact
    truncated SVD, or, given a test matrix Omega [K, l], randomized_svd with
    the same Omega each time.

    Returns dict(q=the final quantize_nf4 result, L1 fp32 [N, r], L2 fp32 [r, K],
    pre=list of pre_t, err=list of err_t,
    plain_err=||W - dequant(quantize(W))|| / ||W|| for comparison)."""
    W = np.asarray(W, np.float32)
    W64 = W.astype(np.float64)
    nW = np.linalg.norm(W64)

    def rank_r(M):
        a, b, _ = truncated_svd(M, r) if Omega is None else randomized_svd(M, Omega, r, power)
        return a.astype(np.float32), b.astype(np.float32)

    plain = float(np.linalg.norm(quant_residual(W, nf4.dequantize_nf4(nf4.quantize_nf4(W, fmt, dq)))
                                 .astype(np.float64)) / nW)
    L1, L2 = rank_r(W)
    pre, errs = [], []
    q = None
    for _ in range(iters):
        q = nf4.quantize_nf4(lowrank_residual(W, L1, L2), fmt, dq)
        Wq_bits = nf4.dequantize_nf4(q)
        Wq = nf4.bf16_bits_to_f32(Wq_bits).reshape(W.shape).astype(np.float64)
        pre.append(float(np.linalg.norm(W64 - Wq - lowrank_product(L1, L2)) / nW))
        L1, L2 = rank_r(quant_residual(W, Wq_bits))
        errs.append(float(np.linalg.norm(W64 - Wq - lowrank_product(L1, L2)) / nW))
    return {"q": q, "L1": L1, "L2": L2, "pre": pre, "err": errs, "plain_err": plain}


def decomposition_error(W: np.ndarray, Wq_bits: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> float:
    """||W - W' - L1 L2||_F / ||W||_F in fp64 (W' from bf16 bits)."""
    W64 = np.asarray(W, np.float32).astype(np.float64)
    Wq = nf4.bf16_bits_to_f32(Wq_bits).reshape(W64.shape).astype(np.float64)
    return float(np.linalg.norm(W64 - Wq - lowrank_product(L1, L2)) / np.linalg.norm(W64))
