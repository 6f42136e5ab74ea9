"""The fused GEMM's stream-K tail against the fp64 oracle.

When the pair tiles do not fill whole waves of cluster slots, the K-steps of
the tiles left after the last full wave are split evenly over the slots; a
tile shared by several clusters is summed from fp32 pieces by whichever CTA
finishes last.  The shapes here make those splits happen in every form:

- a unit inside one tile, and units spanning two and three tiles (with a
  whole tile in the middle), so that tiles are shared by 2 and 3 pieces;
- a piece holding only the adapter K-step, ragged rows and columns in
  shared tiles, one and two accumulators per CTA, forward and dgrad;

and the result is the same bits on every run (the pieces are added in piece
order, whoever finishes last).
"""

import pytest
import torch

import bit_quantized_lora_nf4_b200 as q
import qlora_inputs as qi
from oracle import linear as olin
from tests.gpu_util import TOL, f64, gpu_weight, oracle_weight, rel

pytestmark = pytest.mark.gpu


@pytest.fixture
def always_split(lib):
    """Split every partial last wave, whatever the cost model would choose."""
    prev = q.set_stream_k(q.STREAM_K_ALWAYS)
    yield
    q.set_stream_k(prev)


def _check(case):
    d = qi.make_linear(case)
    _, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    runs = []
    for _ in range(2):
        Y, H = q.linear_fwd(w, X, A, B, d["s"])
        dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H)
        torch.cuda.synchronize()
        assert q.device_status() == 0
        runs.append((Y, dX))
    assert torch.equal(runs[0][0], runs[1][0]) and torch.equal(runs[0][1], runs[1][1])
    Y, dX = runs[0]
    Yr, _ = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    dXr = olin.lora_input_grad(Wd, f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
    errs = {"Y": rel(f64(Y), Yr), "dX": rel(f64(dX), dXr)}
    for k, e in errs.items():
        assert e <= TOL, (k, errs)


@pytest.mark.parametrize("M,N,K,r", [
    (1024, 2048, 1024, 64),   # 16 forward tiles of 17 steps over 17 units: pieces of 2
    (1000, 4000, 512, 64),    # 9-step tiles, 16-step units: units span 3 tiles, ragged rows and columns
    (1024, 4096, 576, 16),    # a unit boundary right before the adapter step
    (480, 1536, 2112, 40),    # one accumulator per CTA (M <= 512), ragged K
    (4096, 1024, 4096, 64),   # more tiles than slots in the dgrad: full waves and a shared tail
])
def test_shared_tiles(always_split, M, N, K, r):
    _check(qi.LinearCase(f"sk_{M}_{N}_{K}_{r}", M, N, K, r, 16.0, 700 + M + N + K + r))


def test_split_chosen_by_the_cost_model(lib):
    """8 forward tiles of 65 K-steps on 74 slots: 32 clusters of ~16 steps
    beat one wave of whole tiles, so the automatic mode splits them."""
    _check(qi.LinearCase("sk_auto", 1024, 1024, 4096, 64, 16.0, 7003))


def test_minimum_workspace_runs_without_the_tail_split(always_split):
    """A workspace of qlora_workspace_min_bytes runs the GEMMs unsplit (the
    last wave partial); both sizes agree with the oracle."""
    case = qi.LinearCase("sk_min", 1024, 2048, 1024, 64, 16.0, 777)
    d = qi.make_linear(case)
    _, Wd = oracle_weight(d["W"])
    w = gpu_weight(d["W"])
    X, A, B, dY = (d[k].cuda() for k in ("X", "A", "B", "dY"))
    lib_ = q.load()
    M, N, K, r = case.M, case.N, case.K, case.r
    outs = {}
    for name, size in (("min", lib_.qlora_workspace_min_bytes), ("full", lib_.qlora_workspace_bytes)):
        wsf = torch.empty(size(q.QLORA_OP_FWD, M, N, K, r), dtype=torch.uint8, device="cuda")
        wsb = torch.empty(size(q.QLORA_OP_BWD, M, N, K, r), dtype=torch.uint8, device="cuda")
        Y, H = q.linear_fwd(w, X, A, B, d["s"], workspace=wsf)
        dX, dA, dB = q.linear_bwd(w, X, dY, A, B, d["s"], H=H, workspace=wsb)
        torch.cuda.synchronize()
        assert q.device_status() == 0
        outs[name] = (Y, dX)
    Yr, _ = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
    dXr = olin.lora_input_grad(Wd, f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
    for name, (Y, dX) in outs.items():
        assert rel(f64(Y), Yr) <= TOL and rel(f64(dX), dXr) <= TOL, name
    # the split changes only the fp32 summation order of the shared tiles
    assert rel(f64(outs["min"][0]), f64(outs["full"][0])) <= 1e-3
