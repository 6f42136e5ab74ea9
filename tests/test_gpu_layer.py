"""A decoder layer with all seven projections on the library (NF4 + LoRA):

- at two reduced widths, output, input gradient and every adapter gradient
  against the fp64 reference layer (oracle/layer.py) built on the oracle's
  dequantized weights: 128 tokens (one-CTA GEMM) and 512 tokens (the CTA-pair
  GEMM that serves the full-size layer);
- at the LLaMA-7B shape with 4 x 2048 tokens (the decoder-layer
  configuration), one forward + backward: finite results, clean device
  status and bit-identical results on a second run.

The layer's glue (RMSNorm, rotary embedding, attention, SwiGLU) runs in torch
with bf16 activations, so the comparison with the fp64 reference carries the
bf16 rounding of every intermediate activation: about 2^-9 relative per
rounding, a few tens of roundings along the longest path, partly cancelling.
Measured at this size: 2.4e-3 on the output and the input gradient, 3.8e-3
to 5.8e-3 on the adapter gradients (relative Frobenius); the tolerance below,
2e-2, is about 3.5 times the largest of them."""

import numpy as np
import pytest
import torch

import qlora_layer as ql
from oracle import layer as olay
from oracle import nf4 as onf4

pytestmark = pytest.mark.gpu

LAYER_TOL = 2e-2


def _rel(a, b):
    a = a.double().cpu()
    b = b.double().cpu()
    return float((a - b).norm() / b.norm())


def _bf16(t):
    return t.to(torch.bfloat16)


# (width, heads, SwiGLU hidden, adapter rank, batch, sequence): 2 x 64 tokens take the
# one-CTA GEMM (M <= 128); 2 x 256 tokens take the CTA-pair kernel with both of its
# TMEM accumulators in use (M > 256), the kernel that serves the full-size layer.
REDUCED = [(512, 4, 1408, 16, 2, 64), (1024, 8, 2816, 64, 2, 256)]


@pytest.mark.parametrize("d,heads,hidden,r,batch,seq", REDUCED, ids=["m128_one_cta", "m512_cta_pair"])
def test_reduced_width_layer_against_the_fp64_reference(lib, d, heads, hidden, r, batch, seq):
    cfg = ql.LayerConfig(d=d, heads=heads, hidden=hidden, r=r)
    params = ql.make_params(cfg, seed=7)
    layer = ql.QLoRADecoderLayer(cfg, params, "cuda")
    g = torch.Generator().manual_seed(8)
    x = _bf16(torch.randn(batch, seq, cfg.d, generator=g))
    gout = _bf16(torch.randn(batch, seq, cfg.d, generator=g))
    xd = x.cuda().requires_grad_(True)
    out = layer(xd)
    (out.float() * gout.cuda().float()).sum().backward()
    torch.cuda.synchronize()

    Wd, A, B = {}, {}, {}
    for name in ql.PROJ:
        oq = onf4.quantize_nf4(params[name + ".W"].numpy())
        Wd[name] = torch.from_numpy(onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64))
        A[name] = _bf16(params[name + ".A"]).double()
        B[name] = _bf16(params[name + ".B"]).double()
    s = layer.proj["q"].s
    ro, rdx, rdA, rdB = olay.layer_fwd_bwd(x.double(), Wd, A, B, s, params["norm1"].double(),
                                           params["norm2"].double(), gout.double(), heads=cfg.heads,
                                           eps=cfg.eps, theta=cfg.rope_theta)
    errs = {"out": _rel(out.detach(), ro), "dx": _rel(xd.grad, rdx)}
    for name in ql.PROJ:
        errs["dA." + name] = _rel(layer.proj[name].A.grad, rdA[name])
        errs["dB." + name] = _rel(layer.proj[name].B.grad, rdB[name])
    print("layer errors", {k: f"{v:.2e}" for k, v in errs.items()})
    bad = {k: v for k, v in errs.items() if not v <= LAYER_TOL}
    assert not bad, errs


def _full_step(layer, x, gout):
    for _, A, B in layer.adapters():
        A.grad = None
        B.grad = None
    xd = x.clone().requires_grad_(True)
    out = layer(xd)
    (out.float() * gout.float()).sum().backward()
    torch.cuda.synchronize()
    return out.detach(), xd.grad.detach(), [(A.grad.clone(), B.grad.clone()) for _, A, B in layer.adapters()]


def test_llama7b_layer_full_shape_runs_and_repeats(lib):
    import bit_quantized_lora_nf4_b200 as q
    cfg = ql.LayerConfig()
    params = ql.make_params(cfg, seed=21)
    layer = ql.QLoRADecoderLayer(cfg, params, "cuda")
    del params
    g = torch.Generator(device="cuda").manual_seed(3)
    x = torch.randn(4, 2048, cfg.d, generator=g, device="cuda").to(torch.bfloat16)
    gout = torch.randn(4, 2048, cfg.d, generator=g, device="cuda").to(torch.bfloat16)
    o1, dx1, gr1 = _full_step(layer, x, gout)
    assert q.device_status() == 0
    assert torch.isfinite(o1).all() and torch.isfinite(dx1).all()
    assert all(torch.isfinite(a).all() and torch.isfinite(b).all() for a, b in gr1)
    o2, dx2, gr2 = _full_step(layer, x, gout)
    assert torch.equal(o1, o2)
    # The library is deterministic: every gradient that does not pass through torch's attention
    # backward (o, gate, up, down) repeats bit for bit.  The fused attention backward accumulates
    # with atomics, so q, k, v and the input gradient only repeat to rounding.
    for name, (a1, b1), (a2, b2) in zip(ql.PROJ, gr1, gr2):
        if name in ("o", "gate", "up", "down"):
            assert torch.equal(a1, a2) and torch.equal(b1, b2), name
        else:
            assert _rel(a1, a2) <= 1e-2 and _rel(b1, b2) <= 1e-2, name
    assert _rel(dx1, dx2) <= 1e-2
