"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the method: it only draws random numbers
and rounds them to the storage dtypes.  Both the CUDA path and the CPU oracle
consume exactly the tensors returned here.

Recipe (one numpy PCG64 generator per case, draws in the fixed order
W, A, B, X, dY, each drawn in fp32 then rounded to nearest-even bf16 where the
tensor is bf16):
  W  [N,K] fp32 ~ N(0, 0.02^2)        frozen base (pretrained weights are close to
                                       Gaussian, the premise of NF4)
  A  [r,K] bf16 ~ N(0, 0.01^2)        adapter down-projection
  B  [N,r] bf16 ~ N(0, 0.01^2)        adapter up-projection
  X  [M,K] bf16 ~ N(0, 1)             activations
  dY [M,N] bf16 ~ N(0, 1)             upstream gradient
  s = alpha / r (fp32).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class LinearCase:
    name: str
    M: int
    N: int
    K: int
    r: int
    alpha: float
    seed: int

    @property
    def s(self) -> float:
        return float(np.float32(self.alpha) / np.float32(self.r))

    def flops_fwd_bwd(self) -> int:
        """Algorithmic flops of fwd+bwd: 2MNK (fwd base) + 2MNK (dgrad base)
        + fwd LoRA 2Mr(K+N) + bwd LoRA 4Mr(K+N) (G, dB, G A, dA)."""
        M, N, K, r = self.M, self.N, self.K, self.r
        return 4 * M * N * K + 6 * M * r * (K + N)


# The single small linear (256x256, r=8, alpha=16, 64 tokens, seed 0).
SMALL = LinearCase("single_linear_256x256_r8_m64", 64, 256, 256, 8, 16.0, 0)

# LLaMA-7B-shaped projections, 4096 tokens (batch 4 x seq 1024), r=64, alpha=16.
LLAMA7B = (
    LinearCase("llama7b_q_4096x4096_m4096", 4096, 4096, 4096, 64, 16.0, 1),
    LinearCase("llama7b_up_11008x4096_m4096", 4096, 11008, 4096, 64, 16.0, 2),
    LinearCase("llama7b_down_4096x11008_m4096", 4096, 4096, 11008, 64, 16.0, 3),
)

# LLaMA-65B-shaped projections, 8192 tokens.
LLAMA65B = (
    LinearCase("llama65b_q_8192x8192_m8192", 8192, 8192, 8192, 64, 16.0, 4),
    LinearCase("llama65b_up_22016x8192_m8192", 8192, 22016, 8192, 64, 16.0, 5),
    LinearCase("llama65b_down_8192x22016_m8192", 8192, 8192, 22016, 64, 16.0, 6),
)

# Decode-style token counts for the dequant-GEMV path.
GEMV_TOKENS = (1, 4, 16)


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def make_linear(case: LinearCase, with_dy: bool = True, M: int | None = None) -> dict:
    """Draw (W, A, B, X, dY) for a case on the host.  ``M`` overrides the token
    count (the GEMV cases reuse the weights of a projection case)."""
    rng = np.random.default_rng(case.seed)
    N, K, r = case.N, case.K, case.r
    M = case.M if M is None else M
    W = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    A = rng.standard_normal((r, K), dtype=np.float32) * np.float32(0.01)
    B = rng.standard_normal((N, r), dtype=np.float32) * np.float32(0.01)
    X = rng.standard_normal((M, K), dtype=np.float32)
    out = {"W": torch.from_numpy(W), "A": _bf16(A), "B": _bf16(B), "X": _bf16(X),
           "s": case.s, "M": M, "N": N, "K": K, "r": r}
    if with_dy:
        out["dY"] = _bf16(rng.standard_normal((M, N), dtype=np.float32))
    return out


def make_weight(n_rows: int, n_cols: int, seed: int, std: float = 0.02) -> torch.Tensor:
    """Gaussian fp32 weight matrix (first draw of the case's generator)."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((n_rows, n_cols), dtype=np.float32) * np.float32(std))


def make_lowrank_weight(n_rows: int, n_cols: int, rank: int, seed: int, std: float = 0.02,
                        strength: tuple = (4.0, 1.5)) -> torch.Tensor:
    """Gaussian fp32 weight plus a planted rank-`rank` component, the structure a
    low-rank plus quantized decomposition looks for.  Draw order: the Gaussian
    [n_rows, n_cols] (scaled by std), then two Gaussian [n, rank] matrices whose
    orthonormal bases (library QR, fp64) give the singular vectors.  The planted
    singular values fall linearly from strength[0] to strength[1] times
    std (sqrt(n_rows) + sqrt(n_cols)), the largest singular value of the
    Gaussian part, so every planted direction stands out of it."""
    rng = np.random.default_rng(seed)
    G = rng.standard_normal((n_rows, n_cols), dtype=np.float32) * np.float32(std)
    U, _ = np.linalg.qr(rng.standard_normal((n_rows, rank)))
    V, _ = np.linalg.qr(rng.standard_normal((n_cols, rank)))
    edge = std * (np.sqrt(n_rows) + np.sqrt(n_cols))
    s = edge * np.linspace(strength[0], strength[1], rank)
    return torch.from_numpy((G.astype(np.float64) + (U * s) @ V.T).astype(np.float32))


def make_test_matrix(n_cols: int, width: int, seed: int) -> torch.Tensor:
    """The Gaussian test matrix [n_cols, width] fp32 a randomized range finder
    draws (passed in as an input, so both sides use the same numbers)."""
    rng = np.random.default_rng(seed)
    return torch.from_numpy(rng.standard_normal((n_cols, width), dtype=np.float32))
