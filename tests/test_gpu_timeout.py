"""The timeout path of the kernels' bounded waits, forced on the device.

Every pipeline wait in the library gives up after qlora_set_wait_limit()
cycles, latches QLORA_ERR_DEVICE_TIMEOUT, lets its issued copies and tensor-core
products land, frees its tensor memory and exits.  With the limit set to 0
the first wait that is not already satisfied gives up; the call must then
report the timeout, and with the default limit restored the next call must
run normally and match the oracle (the context is intact).  Nothing here
faults or hangs the GPU: every wait, including the teardown drains, is bounded.
(The dequantizer's waits are satisfied within one hardware try-wait, so a zero
limit does not reach its timeout branch; tests/test_gpu_status.py drives the
same bounded-wait helper on a barrier that is never signalled.)"""

import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from tests.gpu_util import TOL, f64, gpu_weight, oracle_weight, rel

pytestmark = pytest.mark.gpu

CASES = [
    qi.LinearCase("timeout_pair", 320, 1032, 4096, 64, 16.0, 120),    # CTA-pair fused GEMM, stream-K tail
    qi.LinearCase("timeout_one_cta", 96, 520, 4096, 16, 16.0, 121),  # one-CTA fused GEMM
    qi.LinearCase("timeout_gemv", 4, 2048, 4096, 64, 16.0, 122),     # few-token forward
]


def _run(w, d, case, backward):
    X, A, B = d["X"].cuda(), d["A"].cuda(), d["B"].cuda()
    Y, H = q.linear_fwd(w, X, A, B, case.s)
    if backward:
        q.linear_bwd(w, X, d["dY"].cuda(), A, B, case.s, H=H)
    return Y, H


@pytest.mark.parametrize("case", CASES, ids=lambda c: c.name)
def test_zero_wait_limit_latches_timeout_and_the_context_survives(lib, case):
    d = qi.make_linear(case)
    oq, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    old = q.set_wait_limit(0)
    try:
        for _ in range(3):
            _run(w, d, case, backward=case.M > 16)
        torch.cuda.synchronize()
        st = q.device_status()
    finally:
        q.set_wait_limit(old)
    assert st == 5, q.STATUS_NAMES.get(st, st)          # QLORA_ERR_DEVICE_TIMEOUT
    # the default limit again: a normal call, checked against the oracle
    Y, H = _run(w, d, case, backward=False)
    torch.cuda.synchronize()
    assert q.device_status() == 0
    Yr, Hr = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    assert rel(f64(Y), Yr) <= TOL and rel(f64(H), Hr) <= TOL
