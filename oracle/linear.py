"""Oracle: the LoRA linear on a frozen dequantized base, forward and backward, fp64.

TEST INFRASTRUCTURE ONLY -- see the package docstring.

Shapes (row-major):  X [M,K], W' [N,K] (out x in, the dequantized frozen base),
A [r,K], B [N,r], dY [M,N];  s = alpha / r.

Forward ([Blog-mem]: freeze the pretrained weights and train small low-rank
adapters alongside them; the 4-bit base is dequantized to 16-bit for the pass):
    H  = X A^T                      [M,r]
    Y  = X W'^T + s H B^T           [M,N]
Backward ([QLoRA-abs]: gradients flow through the frozen 4-bit model into the
adapters; [Blog-mem]: gradients flow through the dequantized weights into the
adapters, the base never changes -> no gradient for W'):
    G  = s dY B                     [M,r]
    dX = dY W' + G A                [M,K]
    dA = G^T X                      [r,K]
    dB = s dY^T H                   [N,r]
The backward is the chain rule of the forward; the pages give no formula.

All inputs are converted exactly to fp64 (bf16 and fp32 values are exactly
representable); every product and sum is fp64, so the result is the exact
value of the formula up to fp64 rounding (~1e-16 relative).
"""

from __future__ import annotations

import numpy as np


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def lora_linear_fwd(Wd, X, A, B, s):
    """Returns (Y, H) in fp64."""
    Wd, X, A, B = _f64(Wd), _f64(X), _f64(A), _f64(B)
    s = float(np.float32(s))
    H = X @ A.T
    Y = X @ Wd.T + s * (H @ B.T)
    return Y, H


def lora_input_grad(Wd, dY, A, B, s):
    """dX = dY W' + (s dY B) A.  Row m of dX depends only on row m of dY."""
    Wd, dY, A, B = _f64(Wd), _f64(dY), _f64(A), _f64(B)
    s = float(np.float32(s))
    G = s * (dY @ B)
    return dY @ Wd + G @ A


def lora_adapter_grads(X, dY, A, B, s):
    """(dA, dB) = ((s dY B)^T X, s dY^T (X A^T)): the gradients of the trainable adapters."""
    X, dY, A, B = _f64(X), _f64(dY), _f64(A), _f64(B)
    s = float(np.float32(s))
    H = X @ A.T
    G = s * (dY @ B)
    return G.T @ X, s * (dY.T @ H)


def lora_linear_bwd(Wd, X, dY, A, B, s):
    """Returns (dX, dA, dB) in fp64; W' receives no gradient."""
    dX = lora_input_grad(Wd, dY, A, B, s)
    dA, dB = lora_adapter_grads(X, dY, A, B, s)
    return dX, dA, dB


def rel_frobenius(got, ref) -> float:
    """||got - ref||_F / ||ref||_F in fp64 (0 when both are zero)."""
    g, r = _f64(got), _f64(ref)
    den = np.linalg.norm(r)
    num = np.linalg.norm(g - r)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return float(num / den)
