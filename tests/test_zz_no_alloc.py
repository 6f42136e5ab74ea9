"""qlora_linear_fwd_noalloc: the forward for callers that cannot allocate
device memory (no workspace argument; the scratch is an array inside the
library).  Its output must match the ordinary entry point, qlora_linear_fwd,
within the parity tolerance, on two calls in a row with different shapes, so
that contents left in the shared scratch by the first call cannot leak into
the second.  This file is collected last on purpose."""

import ctypes

import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from tests.gpu_util import TOL, f64, rel

pytestmark = pytest.mark.gpu


def _noalloc(w, X, A, B, s, Y, H):
    lib = q.load()
    st = w.c_struct()
    return lib.qlora_linear_fwd_noalloc(ctypes.byref(st), ctypes.c_void_p(X.data_ptr()), X.shape[0],
                                        ctypes.c_void_p(A.data_ptr()), ctypes.c_void_p(B.data_ptr()), A.shape[0],
                                        s, ctypes.c_void_p(Y.data_ptr()),
                                        None if H is None else ctypes.c_void_p(H.data_ptr()),
                                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_case(case: qi.LinearCase):
    d = qi.make_linear(case, with_dy=False)
    w = q.quantize_nf4(d["W"].cuda())
    X, A, B = d["X"].cuda(), d["A"].cuda(), d["B"].cuda()
    Y_ref, H_ref = q.linear_fwd(w, X, A, B, case.s)            # existing entry point (caller workspace)
    Y = torch.full_like(Y_ref, float("nan"))
    H = torch.full_like(H_ref, float("nan"))
    assert _noalloc(w, X, A, B, case.s, Y, H) == 0
    torch.cuda.synchronize()
    assert q.device_status() == 0
    assert rel(f64(Y), f64(Y_ref)) <= TOL
    assert rel(f64(H), f64(H_ref)) <= TOL


def test_noalloc_matches_workspace_entry_twice(lib):
    # first call: tensor-core path; second call: a different shape, few-token path
    _check_case(qi.LinearCase("noalloc_a", 640, 1032, 1152, 64, 16.0, 71))
    _check_case(qi.LinearCase("noalloc_b", 5, 776, 2112, 24, 16.0, 72))
    # and once more on the first shape after the second has overwritten the scratch
    _check_case(qi.LinearCase("noalloc_a", 640, 1032, 1152, 64, 16.0, 71))


def test_noalloc_rejects_sizes_beyond_the_static_scratch(lib):
    lib_ = q.load()
    w = q.NF4Weight.empty(4096, 4096)
    X = torch.empty((8192, 4096), dtype=torch.bfloat16, device="cuda")
    A = torch.empty((256, 4096), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((4096, 256), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((8192, 4096), dtype=torch.bfloat16, device="cuda")
    assert lib_.qlora_workspace_bytes(q.QLORA_OP_FWD, 8192, 4096, 4096, 256) > (8 << 20)
    assert _noalloc(w, X, A, B, 0.25, Y, None) == 7          # QLORA_ERR_WORKSPACE, nothing launched


def test_noalloc_documented_size_limits(lib):
    """The limits the header states: at r = 64, M = 2048 fits the static
    scratch and M = 4096 does not (the minimum forward workspace grows with
    M r, not with N or K).  The fitting case runs and matches the workspace
    entry point; the other is refused before anything is enqueued."""
    lib_ = q.load()
    limit = q.QLORA_STATIC_SCRATCH_BYTES
    assert lib_.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 2048, 4096, 4096, 64) <= limit
    assert lib_.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 3413, 4096, 4096, 64) <= limit
    assert lib_.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 3414, 4096, 4096, 64) > limit
    assert lib_.qlora_workspace_min_bytes(q.QLORA_OP_FWD, 4096, 4096, 4096, 64) > limit
    # fits: runs, and equals the ordinary entry point within the parity tolerance
    _check_case(qi.LinearCase("noalloc_fits", 2048, 4096, 4096, 64, 16.0, 73))
    # does not fit: QLORA_ERR_WORKSPACE, outputs untouched
    w = q.NF4Weight.empty(4096, 4096)
    X = torch.zeros((4096, 4096), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((64, 4096), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((4096, 64), dtype=torch.bfloat16, device="cuda")
    Y = torch.full((4096, 4096), 7.0, dtype=torch.bfloat16, device="cuda")
    assert _noalloc(w, X, A, B, 0.25, Y, None) == 7
    torch.cuda.synchronize()
    assert bool((Y == 7.0).all())
