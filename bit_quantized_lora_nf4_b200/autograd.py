"""torch.autograd wiring of the library's linear (argument marshalling only).

QLoRALinear holds a frozen 4-bit base weight and trainable bf16 adapters A
[r, K], B [N, r]; forward and backward run qlora_linear_fwd / qlora_linear_bwd
("QLoRA: fine-tuning a 65B model on one GPU", section "Where the memory goes":
gradients flow through the dequantized frozen weights into the adapters, the
base itself gets no gradient).  Inputs of any leading shape are flattened to
[tokens, K]; workspaces are cached per token count.
"""

from __future__ import annotations

import torch

from . import NF4Weight, linear_bwd, linear_fwd, quantize_nf4, workspace_bytes, QLORA_OP_BWD, QLORA_OP_FWD


class _LinearFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x2, A, B, mod):
        Y, H = linear_fwd(mod.weight, x2, A, B, mod.s, workspace=mod._ws(QLORA_OP_FWD, x2.shape[0]))
        ctx.save_for_backward(x2, A, B, H)
        ctx.mod = mod
        return Y

    @staticmethod
    def backward(ctx, dY):
        x2, A, B, H = ctx.saved_tensors
        mod = ctx.mod
        dX, dA, dB = linear_bwd(mod.weight, x2, dY.contiguous(), A, B, mod.s, H=H,
                                workspace=mod._ws(QLORA_OP_BWD, x2.shape[0]))
        return dX, dA.to(A.dtype), dB.to(B.dtype), None


class QLoRALinear(torch.nn.Module):
    """y = x W'^T + s (x A^T) B^T with W' the dequantized frozen base."""

    def __init__(self, weight: NF4Weight, A: torch.Tensor, B: torch.Tensor, alpha: float):
        super().__init__()
        self.weight = weight
        self.A = torch.nn.Parameter(A.to(torch.bfloat16).contiguous())
        self.B = torch.nn.Parameter(B.to(torch.bfloat16).contiguous())
        r = A.shape[0]
        self.s = float(torch.tensor(alpha, dtype=torch.float32) / torch.tensor(r, dtype=torch.float32))
        self._wss = {}

    @classmethod
    def from_float(cls, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor, alpha: float, format: int = 0):
        """Quantize an fp32 or bf16 weight [N, K] (on its device) and wrap it with adapters."""
        Wq = W.contiguous() if W.dtype in (torch.float32, torch.bfloat16) else W.float().contiguous()
        return cls(quantize_nf4(Wq, format=format), A, B, alpha)

    def _ws(self, op: int, M: int) -> torch.Tensor:
        key = (op, M)
        ws = self._wss.get(key)
        if ws is None:
            n = workspace_bytes(op, M, self.weight.rows, self.weight.cols, self.A.shape[0])
            ws = torch.empty(n, dtype=torch.uint8, device=self.A.device)
            self._wss[key] = ws
        return ws

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, x.shape[-1]).to(torch.bfloat16).contiguous()
        y = _LinearFn.apply(x2, self.A, self.B, self)
        return y.reshape(*lead, self.weight.rows)
