"""Device-side failure reporting without faulting the GPU: a bounded wait on a
barrier nothing signals gives up and latches QLORA_ERR_DEVICE_TIMEOUT, and the
context stays usable afterwards."""

import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out(lib):
    assert q.device_status() == 0
    assert q.selftest_wait_timeout(200000) == 5      # ~0.1 ms bound
    assert q.device_status() == 0
    # the context still works
    w = q.quantize_nf4(qi.make_weight(64, 256, seed=1).cuda())
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert w.codes.numel() == 64 * 256 // 2
