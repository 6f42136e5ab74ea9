"""The backward's dB and dA products run on a side stream beside the dgrad
GEMM.  The results must not depend on it: the same call with the timing hook
on (every launch on the caller's stream), and the same call replayed from a
CUDA graph (the fork and join captured), give the same bits."""

import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,N,K,r", [(512, 1024, 1024, 64), (4096, 4096, 4096, 64), (300, 1032, 1152, 32)])
def test_side_stream_changes_no_bits(lib, M, N, K, r):
    case = qi.LinearCase(f"side_{M}_{N}_{K}", M, N, K, r, 16.0, 1000 + M + N)
    d = qi.make_linear(case)
    w = q.quantize_nf4(d["W"].cuda())
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    _, H = q.linear_fwd(w, X, A, B, d["s"])
    g_side = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    q.profile_enable(True)
    g_seq = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
    torch.cuda.synchronize()
    q.profile_enable(False)
    assert q.device_status() == 0
    for a, b in zip(g_side, g_seq):
        assert torch.equal(a, b)
    # captured: the side stream's fork and join become graph edges
    outs = tuple(torch.empty_like(t) for t in g_side)
    ws = torch.empty(q.workspace_bytes(q.QLORA_OP_BWD, M, N, K, r), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        q.linear_bwd(w, X, dY, A, B, d["s"], H=H, outs=outs, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        q.linear_bwd(w, X, dY, A, B, d["s"], H=H, outs=outs, workspace=ws)
    for t in outs:
        t.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert q.device_status() == 0
    for a, b in zip(outs, g_seq):
        assert torch.equal(a, b)
    del graph
