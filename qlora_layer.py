"""A LLaMA-7B-shaped decoder layer whose seven projections are the library's
NF4 + LoRA linears; the rest (RMSNorm, rotary position embedding, causal
attention, SwiGLU) is plain torch glue.  Used by the bench and the layer
tests; the glue is not part of the library.

Shapes of the layer ("QLoRA: efficient finetuning of quantized LLMs",
Abstract, and the LLaMA models the pages finetune): d = 4096, 32 heads of
128, SwiGLU hidden 11008, RMSNorm before attention and before the MLP,
residual connections.  q, k, v, o (4096 x 4096), gate, up (11008 x 4096) and
down (4096 x 11008) are frozen NF4 with trainable rank-r adapters; the norm
weights are frozen.

Synthetic parameters: one seeded generator per layer, drawn in the order q,
k, v, o, gate, up, down (each: W ~ N(0, 0.02^2) fp32, A, B ~ N(0, 0.01^2)),
then the two norm weights (1 + N(0, 0.02^2)).
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import bit_quantized_lora_nf4_b200 as q
from bit_quantized_lora_nf4_b200.autograd import QLoRALinear

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class LayerConfig:
    d: int = 4096
    heads: int = 32
    hidden: int = 11008
    r: int = 64
    alpha: float = 16.0
    eps: float = 1e-5
    rope_theta: float = 10000.0

    def shapes(self):
        d, h = self.d, self.hidden
        return {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d), "gate": (h, d), "up": (h, d), "down": (d, h)}

    def linear_flops_fwd_bwd(self, tokens: int) -> int:
        """4 M N K + 6 M r (K + N) summed over the seven projections."""
        return sum(4 * tokens * n * k + 6 * tokens * self.r * (k + n) for n, k in self.shapes().values())


def make_params(cfg: LayerConfig, seed: int) -> dict:
    """fp32 host tensors of the layer (see the module docstring for the recipe)."""
    rng = np.random.default_rng(seed)
    p = {}
    for name in PROJ:
        n, k = cfg.shapes()[name]
        p[name + ".W"] = torch.from_numpy(rng.standard_normal((n, k), dtype=np.float32) * np.float32(0.02))
        p[name + ".A"] = torch.from_numpy(rng.standard_normal((cfg.r, k), dtype=np.float32) * np.float32(0.01))
        p[name + ".B"] = torch.from_numpy(rng.standard_normal((n, cfg.r), dtype=np.float32) * np.float32(0.01))
    for name in ("norm1", "norm2"):
        p[name] = torch.from_numpy(1 + rng.standard_normal(cfg.d, dtype=np.float32) * np.float32(0.02))
    return p


def rope_tables(cfg: LayerConfig, seq: int, device) -> tuple[torch.Tensor, torch.Tensor]:
    hd = cfg.d // cfg.heads
    inv = 1.0 / (cfg.rope_theta ** (torch.arange(0, hd, 2, dtype=torch.float32, device=device) / hd))
    ang = torch.arange(seq, dtype=torch.float32, device=device)[:, None] * inv[None, :]
    return torch.cos(ang), torch.sin(ang)


def apply_rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """x [b, h, s, hd]: rotate the pairs (x[..., :hd/2], x[..., hd/2:])."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h].float(), x[..., h:].float()
    return torch.cat([x1 * cos - x2 * sin, x2 * cos + x1 * sin], dim=-1).to(x.dtype)


class QLoRADecoderLayer(torch.nn.Module):
    def __init__(self, cfg: LayerConfig, params: dict, device, format: int = q.FORMAT_NF4):
        super().__init__()
        self.cfg = cfg
        self.proj = torch.nn.ModuleDict({
            name: QLoRALinear.from_float(params[name + ".W"].to(device), params[name + ".A"].to(device),
                                         params[name + ".B"].to(device), cfg.alpha, format)
            for name in PROJ})
        self.register_buffer("norm1", params["norm1"].to(device))
        self.register_buffer("norm2", params["norm2"].to(device))

    def _rms(self, x: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
        xf = x.float()
        return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + self.cfg.eps) * w).to(torch.bfloat16)

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        b, s, d = x.shape
        hn, hd = self.cfg.heads, d // self.cfg.heads
        p = self.proj
        n1 = self._rms(x, self.norm1)
        qh = p["q"](n1).view(b, s, hn, hd).transpose(1, 2)
        kh = p["k"](n1).view(b, s, hn, hd).transpose(1, 2)
        vh = p["v"](n1).view(b, s, hn, hd).transpose(1, 2)
        cos, sin = rope_tables(self.cfg, s, x.device)
        qh, kh = apply_rope(qh, cos, sin), apply_rope(kh, cos, sin)
        att = torch.nn.functional.scaled_dot_product_attention(qh, kh, vh, is_causal=True)
        h = x + p["o"](att.transpose(1, 2).reshape(b, s, d))
        n2 = self._rms(h, self.norm2)
        mlp = p["down"](torch.nn.functional.silu(p["gate"](n2)) * p["up"](n2))
        return h + mlp

    def adapters(self):
        return [(name, self.proj[name].A, self.proj[name].B) for name in PROJ]
