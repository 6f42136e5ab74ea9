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
