"""fp64 CPU reference of a LLaMA-shaped decoder layer with QLoRA linears.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).  Plain PyTorch CPU ops in
fp64; gradients by torch autograd in fp64.  Shares no code with the GPU layer
harness.

Sources: [QLoRA-abs] (LLaMA models finetuned through frozen 4-bit bases into
LoRA adapters; only the adapters are trained), [Blog-mem] (the base is
dequantized inside each forward and backward pass).  The layer around the
linears is the LLaMA block, a reading (the pages give no layer code):
    h   = x + o( attn( rope(q(n1)), rope(k(n1)), v(n1) ) ),   n1 = rms(x) * w1
    out = h + down( silu(gate(n2)) * up(n2) ),                 n2 = rms(h) * w2
with rms(z) = z / sqrt(mean(z^2) + eps), causal softmax attention scaled by
1/sqrt(head_dim), rotary embedding on pairs (j, j + head_dim/2) with angle
pos / theta^(2j/head_dim).  Each linear is y = z W'^T + s (z A^T) B^T with W'
the dequantized (bf16) base, as in oracle.linear.lora_linear_fwd.
"""

from __future__ import annotations

import math

import torch

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


def lora_linear(z, W, A, B, s):
    """z W^T + s (z A^T) B^T (the method's linear, fp64)."""
    return z @ W.T + s * ((z @ A.T) @ B.T)


def rms_norm(z, w, eps):
    return z / torch.sqrt((z * z).mean(-1, keepdim=True) + eps) * w


def rope(x, theta):
    """x [b, h, s, hd]: pairs (j, j + hd/2) rotated by pos / theta^(2j / hd)."""
    hd = x.shape[-1]
    half = hd // 2
    j = torch.arange(half, dtype=torch.float64)
    inv = theta ** (-2.0 * j / hd)
    ang = torch.arange(x.shape[-2], dtype=torch.float64)[:, None] * inv[None, :]
    c, s_ = torch.cos(ang), torch.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return torch.cat([x1 * c - x2 * s_, x2 * c + x1 * s_], dim=-1)


def causal_attention(qh, kh, vh):
    """softmax(Q K^T / sqrt(hd) with future positions masked) V, per head."""
    hd = qh.shape[-1]
    scores = (qh @ kh.transpose(-1, -2)) / math.sqrt(hd)
    sq = scores.shape[-1]
    mask = torch.triu(torch.ones(sq, sq, dtype=torch.bool), diagonal=1)
    scores = scores.masked_fill(mask, float("-inf"))
    return torch.softmax(scores, dim=-1) @ vh


def layer_forward(x, Wd, A, B, s, norm1, norm2, heads, eps, theta):
    b, sq, d = x.shape
    hd = d // heads
    n1 = rms_norm(x, norm1, eps)
    qh = lora_linear(n1, Wd["q"], A["q"], B["q"], s).view(b, sq, heads, hd).transpose(1, 2)
    kh = lora_linear(n1, Wd["k"], A["k"], B["k"], s).view(b, sq, heads, hd).transpose(1, 2)
    vh = lora_linear(n1, Wd["v"], A["v"], B["v"], s).view(b, sq, heads, hd).transpose(1, 2)
    att = causal_attention(rope(qh, theta), rope(kh, theta), vh)
    h = x + lora_linear(att.transpose(1, 2).reshape(b, sq, d), Wd["o"], A["o"], B["o"], s)
    n2 = rms_norm(h, norm2, eps)
    g = lora_linear(n2, Wd["gate"], A["gate"], B["gate"], s)
    u = lora_linear(n2, Wd["up"], A["up"], B["up"], s)
    return h + lora_linear(g * torch.sigmoid(g) * u, Wd["down"], A["down"], B["down"], s)


def layer_fwd_bwd(x, Wd, A, B, s, norm1, norm2, g_out, heads=32, eps=1e-5, theta=10000.0):
    """Output, input gradient and adapter gradients for the upstream gradient
    g_out (loss = sum(out * g_out)); all fp64 CPU tensors in, fp64 out."""
    x = x.detach().clone().requires_grad_(True)
    A = {k: v.detach().clone().requires_grad_(True) for k, v in A.items()}
    B = {k: v.detach().clone().requires_grad_(True) for k, v in B.items()}
    out = layer_forward(x, Wd, A, B, s, norm1, norm2, heads, eps, theta)
    (out * g_out).sum().backward()
    return (out.detach(), x.grad.detach(), {k: A[k].grad.detach() for k in PROJ},
            {k: B[k].grad.detach() for k in PROJ})
