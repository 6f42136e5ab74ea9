"""GPU parity of the quantizer and dequantizer against the oracle: bit-exact
codes, 8-bit constants, fp32 group scales and bf16 dequantized weights."""

import numpy as np
import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import nf4 as onf4
from tests.gpu_util import assert_weight_bits, gpu_weight

pytestmark = pytest.mark.gpu


def _roundtrip(W: torch.Tensor):
    w = gpu_weight(W)
    oq = onf4.quantize_nf4(W.numpy())
    assert_weight_bits(w, oq)
    deq = q.dequantize(w)
    torch.cuda.synchronize()
    got = deq.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    exp = onf4.dequantize_nf4(oq).reshape(-1)
    assert np.array_equal(got, exp), "dequantized bf16 differs"


def test_small_config_bit_exact(lib):
    _roundtrip(qi.make_linear(qi.SMALL)["W"])


@pytest.mark.parametrize("shape", [(64, 64), (3, 5), (1, 1), (7, 4096 * 4 + 1000), (256 * 64 + 64, 1),
                                   (33, 1000)])
def test_ragged_and_partial_groups(lib, shape):
    W = qi.make_weight(*shape, seed=sum(shape))
    _roundtrip(W)


def test_special_values(lib):
    W = qi.make_weight(64, 512, seed=3)
    W[0, :64] = 0.0                               # all-zero block
    W[1, :64] = -0.0
    W[2, 5] = 1e30                                # huge absmax
    W[3, :] = 1e-40                               # subnormal weights
    W[4, :64] = torch.linspace(-1, 1, 64)         # exact endpoints
    v = torch.from_numpy(onf4.nf4_codebook())
    W[5, :64] = v.repeat(4) * 3.0                 # grid values
    _roundtrip(W)


def test_nonfinite_latches_status(lib):
    W = qi.make_weight(16, 1024, seed=4)
    W[3, 7] = float("nan")
    q.quantize_nf4(W.cuda())
    assert q.device_status() == 4
    assert q.device_status() == 0                 # cleared on read


@pytest.mark.parametrize("case", qi.LLAMA7B, ids=lambda c: c.name)
def test_llama7b_weights_bit_exact(lib, case):
    _roundtrip(qi.make_weight(case.N, case.K, case.seed))


# --------------------------------------------------------------------------- ties to the lower index

def _threshold_probes(levels: np.ndarray, a: np.float32, span: int = 3) -> list:
    """Weights w whose normalised value fl32(w / a) lands on every decision
    threshold of the table and `span` fp32 steps either side of it.  For a
    power-of-two a, w = m a is exact, so n equals each probe m; m runs over the
    fp32 values around the exact midpoint of every pair of neighbouring levels
    (where the midpoint is itself an fp32 value, n sits exactly on the tie).
    For other a, w = fl32(m a) and its neighbours, which put n on, or one
    rounding away from, the same values."""
    out = []
    for i in range(15):
        mid = (np.float64(levels[i]) + np.float64(levels[i + 1])) / 2
        m = np.float32(mid)
        vals = [m]
        lo = hi = m
        for _ in range(span):
            lo = np.nextafter(lo, np.float32(-2))
            hi = np.nextafter(hi, np.float32(2))
            vals += [lo, hi]
        for v in vals:
            w = np.float32(v * a)
            out += [w, np.nextafter(w, np.float32(-1)), np.nextafter(w, np.float32(1))] if (a != 1.0 and
                                                                                              np.log2(a) % 1) else [w]
    return out


def _tie_weight(levels: np.ndarray) -> torch.Tensor:
    blocks = []
    for a in (np.float32(1.0), np.float32(2.0 ** -6), np.float32(2.0 ** -11), np.float32(0.0371),
              np.float32(0.00713)):
        probes = [p for p in _threshold_probes(levels, a) if abs(p) < a]
        for j in range(0, len(probes), 63):
            chunk = probes[j:j + 63]
            blk = np.zeros(64, np.float32)
            blk[0] = a if (j // 63) % 2 == 0 else -a          # the block's absmax, either sign
            blk[1:1 + len(chunk)] = chunk
            blocks.append(blk)
    W = np.concatenate(blocks)
    pad = (-W.size) % 256
    W = np.concatenate([W, np.zeros(pad, np.float32)])
    return torch.from_numpy(W.reshape(-1, 256).copy())


@pytest.mark.parametrize("fmt,fid", [("nf4", q.FORMAT_NF4), ("fp4", q.FORMAT_FP4), ("int4", q.FORMAT_INT4)])
def test_ties_break_to_the_lower_index(lib, fmt, fid):
    """Each normalized weight takes the nearest level ("QLoRA: fine-tuning a 65B
    model on one GPU", section "NormalFloat, double quantization, paged
    optimizers"), an exact tie going to the lower code index.  Every
    threshold of every table is hit exactly (the midpoints that are fp32 values
    give true ties: e.g. half of the first level above zero) and one to three
    fp32 steps either side; the codes must equal the oracle's bit for bit."""
    lv = onf4.codebook(fmt)
    W = _tie_weight(lv)
    oq = onf4.quantize_nf4(W.numpy(), fmt)
    n = onf4.normalize(W.numpy().ravel(), onf4.block_absmax(W.numpy().ravel()))
    exact_ties = sum(1 for i in range(15) if lv[i] != lv[i + 1]
                     and np.float64(np.float32((np.float64(lv[i]) + np.float64(lv[i + 1])) / 2))
                     == (np.float64(lv[i]) + np.float64(lv[i + 1])) / 2)
    assert exact_ties >= 1
    w = q.quantize_nf4(W.cuda().contiguous(), format=fid)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert_weight_bits(w, oq)
    # on the exact ties the code is the lowest index among the nearest levels (the definition, read off directly)
    codes = onf4.unpack_nibbles(oq["codes"], W.numel())
    for i in range(15):
        mid = (np.float64(lv[i]) + np.float64(lv[i + 1])) / 2
        at = np.nonzero(n.astype(np.float64) == mid)[0]
        if lv[i] != lv[i + 1] and at.size:
            d = np.abs(mid - lv.astype(np.float64))
            assert np.all(codes[at] == int(np.nonzero(d == d.min())[0][0])), (fmt, i)


# --------------------------------------------------------------------------- bf16 weights

@pytest.mark.parametrize("shape", [(256, 256), (7, 4096 * 4 + 1000), (33, 1000), (4096, 11008)])
@pytest.mark.parametrize("dq", [q.DQ_PLAIN, q.DQ_SIGNED])
def test_bf16_weights_bit_exact(lib, shape, dq):
    """A bf16 weight quantizes to the same bits as the oracle on its (exact)
    fp32 widening, and as the library's own fp32 call on that widening."""
    W16 = qi.make_weight(*shape, seed=60 + shape[0]).to(torch.bfloat16)
    W32 = W16.float()
    oq = onf4.quantize_nf4(W32.numpy(), dq="signed" if dq == q.DQ_SIGNED else "plain")
    w = q.quantize_nf4(W16.cuda().contiguous(), dq=dq)
    w32 = q.quantize_nf4(W32.cuda().contiguous(), dq=dq)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    if dq == q.DQ_PLAIN:
        assert_weight_bits(w, oq)
    else:   # signed constants: the group scales, then mu, in one array
        assert np.array_equal(w.codes.cpu().numpy(), oq["codes"])
        assert np.array_equal(w.absmax_q.cpu().numpy(), oq["absmax_q"])
        assert np.array_equal(w.scales.cpu().numpy().view(np.uint32), oq["group_scale"].view(np.uint32))
        assert w.offset.cpu().numpy().view(np.uint32)[0] == np.float32(oq["offset"]).view(np.uint32)
    assert torch.equal(w.codes, w32.codes) and torch.equal(w.absmax_q, w32.absmax_q)
    assert torch.equal(w.group_scale, w32.group_scale)
    got = q.dequantize(w).view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1)
    assert np.array_equal(got, onf4.dequantize_nf4(oq).reshape(-1))
