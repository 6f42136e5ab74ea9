"""Pins of the fp64 reference decoder layer (oracle/layer.py), on the CPU:
its linear is the oracle linear, its backward matches finite differences,
causal attention lets position 0 see only itself, RMSNorm with unit weights
gives unit root-mean-square, and the rotary embedding is a rotation (norm
preserving) that leaves position 0 unchanged."""

import numpy as np
import torch

from oracle import layer as ol
from oracle import linear as olin


def _tiny(seed=0, b=2, s=5, d=16, heads=2, hidden=24, r=4):
    g = torch.Generator().manual_seed(seed)
    rn = lambda *sh, sc=1.0: torch.randn(*sh, generator=g, dtype=torch.float64) * sc
    shapes = {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d), "gate": (hidden, d), "up": (hidden, d),
              "down": (d, hidden)}
    Wd = {k: rn(*v, sc=0.2) for k, v in shapes.items()}
    A = {k: rn(r, v[1], sc=0.1) for k, v in shapes.items()}
    B = {k: rn(v[0], r, sc=0.1) for k, v in shapes.items()}
    x = rn(b, s, d)
    n1, n2 = 1 + rn(d, sc=0.1), 1 + rn(d, sc=0.1)
    return x, Wd, A, B, n1, n2, heads


def test_linear_is_the_oracle_linear():
    rng = np.random.default_rng(1)
    z, W, A, B = (rng.standard_normal(s) for s in ((7, 12), (9, 12), (3, 12), (9, 3)))
    want, _ = olin.lora_linear_fwd(W, z, A, B, 0.5)
    got = ol.lora_linear(*(torch.from_numpy(t) for t in (z, W, A, B)), 0.5).numpy()
    assert np.allclose(got, want, rtol=1e-13, atol=1e-13)


def test_backward_matches_finite_differences():
    x, Wd, A, B, n1, n2, heads = _tiny()
    g = torch.randn(x.shape, generator=torch.Generator().manual_seed(9), dtype=torch.float64)
    out, dx, dA, dB = ol.layer_fwd_bwd(x, Wd, A, B, 0.25, n1, n2, g, heads=heads)
    f = lambda xx, AA, BB: float((ol.layer_forward(xx, Wd, AA, BB, 0.25, n1, n2, heads, 1e-5, 10000.0) * g).sum())
    eps = 1e-6
    for idx in [(0, 0, 0), (1, 4, 7), (0, 2, 15)]:
        xp, xm = x.clone(), x.clone()
        xp[idx] += eps
        xm[idx] -= eps
        num = (f(xp, A, B) - f(xm, A, B)) / (2 * eps)
        assert abs(num - float(dx[idx])) <= 1e-6 * max(1.0, abs(num))
    for name, idx in [("q", (1, 3)), ("down", (0, 20)), ("v", (3, 0))]:
        Ap = {k: v.clone() for k, v in A.items()}
        Am = {k: v.clone() for k, v in A.items()}
        Ap[name][idx] += eps
        Am[name][idx] -= eps
        num = (f(x, Ap, B) - f(x, Am, B)) / (2 * eps)
        assert abs(num - float(dA[name][idx])) <= 1e-6 * max(1.0, abs(num))
    for name, idx in [("gate", (5, 2)), ("o", (0, 0))]:
        Bp = {k: v.clone() for k, v in B.items()}
        Bm = {k: v.clone() for k, v in B.items()}
        Bp[name][idx] += eps
        Bm[name][idx] -= eps
        num = (f(x, A, Bp) - f(x, A, Bm)) / (2 * eps)
        assert abs(num - float(dB[name][idx])) <= 1e-6 * max(1.0, abs(num))


def test_causal_attention_first_position_sees_only_itself():
    g = torch.Generator().manual_seed(2)
    qh, kh, vh = (torch.randn(1, 2, 6, 8, generator=g, dtype=torch.float64) for _ in range(3))
    out = ol.causal_attention(qh, kh, vh)
    assert torch.allclose(out[..., 0, :], vh[..., 0, :], rtol=0, atol=1e-15)
    # the last position averages all values with softmax weights of the full row
    w = torch.softmax((qh[..., -1:, :] @ kh.transpose(-1, -2)) / np.sqrt(8), dim=-1)
    assert torch.allclose(out[..., -1:, :], w @ vh, rtol=1e-12, atol=1e-12)


def test_rms_norm_and_rope_properties():
    z = torch.randn(3, 4, 32, dtype=torch.float64)
    n = ol.rms_norm(z, torch.ones(32, dtype=torch.float64), 0.0)
    assert torch.allclose(n.pow(2).mean(-1), torch.ones(3, 4, dtype=torch.float64), rtol=1e-12)
    x = torch.randn(1, 2, 7, 16, dtype=torch.float64)
    y = ol.rope(x, 10000.0)
    assert torch.allclose(y[..., 0, :], x[..., 0, :], rtol=0, atol=0)      # angle 0 at position 0
    pair = lambda t: t[..., :8] ** 2 + t[..., 8:] ** 2
    assert torch.allclose(pair(y), pair(x), rtol=1e-12)                     # each pair is rotated
