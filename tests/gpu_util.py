"""Helpers for the GPU parity tests: run the CUDA path through the binding and
the oracle on the same seeded host inputs."""

import numpy as np
import torch

import bit_quantized_lora_nf4_b200 as q
from oracle import linear as olin
from oracle import nf4 as onf4

TOL = 2e-3   # relative Frobenius bound on Y, dX, dA, dB (bf16 inputs, fp32 accumulation)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_weight(W: torch.Tensor):
    """Oracle quantization and its dequantized bf16 weight as fp64."""
    oq = onf4.quantize_nf4(W.numpy())
    Wd = onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64)
    return oq, Wd


def gpu_weight(W: torch.Tensor) -> q.NF4Weight:
    w = q.quantize_nf4(W.cuda().contiguous())
    torch.cuda.synchronize()
    assert q.device_status() == 0
    return w


def assert_weight_bits(w: q.NF4Weight, oq) -> None:
    assert np.array_equal(w.codes.cpu().numpy(), oq["codes"]), "codes differ"
    assert np.array_equal(w.absmax_q.cpu().numpy(), oq["absmax_q"]), "8-bit constants differ"
    assert np.array_equal(w.group_scale.cpu().numpy().view(np.uint32), oq["group_scale"].view(np.uint32)), \
        "group scales differ"


def rel(got, ref) -> float:
    return olin.rel_frobenius(got, ref)
