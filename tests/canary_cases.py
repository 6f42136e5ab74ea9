"""Canary-padded output buffers for the GPU tests (stand-in for a memory
sanitizer, which these tests do not run).

Every output of a library call is carved from a larger buffer with PAD bytes
of a fixed byte pattern on both sides (PAD is a multiple of 16, so the carved
view keeps the library's 16-byte alignment); after the call the pads must be
unchanged.  run_all() drives the quantizer (fp32 and bf16 weights, both block
constant readings), the dequantizer (bulk and ragged tail), the few-token
forward and the tensor-core linear forward and backward on small ragged
shapes, checks the pads, the device status and parity against the oracle, and
returns the outputs so that two builds of the library can be compared bit for
bit.  Run as a script it saves them to the .npz file named on the command line.
"""

from __future__ import annotations

import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bit_quantized_lora_nf4_b200 as q  # noqa: E402
import qlora_inputs as qi  # noqa: E402
from oracle import linear as olin  # noqa: E402
from oracle import nf4 as onf4  # noqa: E402

PAD = 4096
PATTERN = 0xA5
TOL = 2e-3


class Padded:
    """A device tensor of `shape` and `dtype` with PAD canary bytes either side."""

    def __init__(self, shape, dtype, dev="cuda"):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.nbytes = n
        self.raw = torch.full((n + 2 * PAD,), PATTERN, dtype=torch.uint8, device=dev)
        self.t = self.raw[PAD:PAD + n].view(dtype).view(shape)

    def intact(self) -> bool:
        head, tail = self.raw[:PAD], self.raw[PAD + self.nbytes:]
        return bool((head == PATTERN).all()) and bool((tail == PATTERN).all())


def _rel(a, b) -> float:
    return olin.rel_frobenius(a, b)


def _quant_cases(out):
    shapes = [(7, 4096 * 4 + 1000), (256 + 8, 4160), (3, 5), (1, 64)]
    for i, (rows, cols) in enumerate(shapes):
        W32 = qi.make_weight(rows, cols, seed=90 + i)
        for dt, Win in (("f32", W32), ("bf16", W32.to(torch.bfloat16))):
            for dq in (q.DQ_PLAIN, q.DQ_SIGNED):
                w = q.NF4Weight.empty(rows, cols, "cuda", q.FORMAT_NF4, dq)
                codes = Padded(w.codes.shape, torch.uint8)
                absq = Padded(w.absmax_q.shape, torch.uint8)
                gsc = Padded(w.group_scale.shape, torch.float32)
                w = q.NF4Weight(rows, cols, codes.t, absq.t, gsc.t, q.FORMAT_NF4, dq)
                q.quantize_nf4(Win.cuda().contiguous(), out=w)
                deq = Padded((rows, cols), torch.bfloat16)
                q.dequantize(w, out=deq.t)
                torch.cuda.synchronize()
                assert q.device_status() == 0, (rows, cols, dt, dq)
                for name, buf in (("codes", codes), ("absmax_q", absq), ("group_scale", gsc), ("dequant", deq)):
                    assert buf.intact(), f"canary overwritten next to {name} {rows}x{cols} {dt} dq={dq}"
                oq = onf4.quantize_nf4(Win.float().numpy(), dq="signed" if dq == q.DQ_SIGNED else "plain")
                assert np.array_equal(codes.t.cpu().numpy(), oq["codes"])
                assert np.array_equal(deq.t.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1),
                                      onf4.dequantize_nf4(oq).reshape(-1))
                key = f"q_{rows}x{cols}_{dt}_{dq}"
                out[key + "_codes"] = codes.t.cpu().numpy()
                out[key + "_deq"] = deq.t.view(torch.int16).cpu().numpy()


def _linear_cases(out):
    cases = [qi.LinearCase("canary_gemv_1", 1, 776, 2112, 24, 16.0, 95),
             qi.LinearCase("canary_gemv_13", 13, 392, 640, 40, 16.0, 96),
             qi.LinearCase("canary_one_cta", 72, 520, 1088, 16, 16.0, 97),
             qi.LinearCase("canary_pair", 300, 1032, 1152, 64, 16.0, 98)]
    for case in cases:
        d = qi.make_linear(case)
        w = q.quantize_nf4(d["W"].cuda())
        oq, Wd = onf4.quantize_nf4(d["W"].numpy()), None
        Wd = onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64)
        X, A, B, dY = d["X"].cuda(), d["A"].cuda(), d["B"].cuda(), d["dY"].cuda()
        M, N, K, r = case.M, case.N, case.K, case.r
        Y = Padded((M, N), torch.bfloat16)
        H = Padded((M, r), torch.float32)
        q.linear_fwd(w, X, A, B, case.s, out=Y.t, h_out=H.t)
        bufs = {"Y": Y, "H": H}
        if M > 16:   # the backward runs the tensor-core kernels at every M; the GEMV cases cover M <= 16 forward
            dX = Padded((M, K), torch.bfloat16)
            dA = Padded((r, K), torch.float32)
            dB = Padded((N, r), torch.float32)
            q.linear_bwd(w, X, dY, A, B, case.s, H=H.t, outs=(dX.t, dA.t, dB.t))
            bufs.update({"dX": dX, "dA": dA, "dB": dB})
        torch.cuda.synchronize()
        assert q.device_status() == 0, case.name
        for name, buf in bufs.items():
            assert buf.intact(), f"canary overwritten next to {name} in {case.name}"
        f64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)  # noqa: E731
        Yr, Hr = olin.lora_linear_fwd(Wd, f64(d["X"]), f64(d["A"]), f64(d["B"]), d["s"])
        assert _rel(f64(Y.t), Yr) <= TOL and _rel(f64(H.t), Hr) <= TOL, case.name
        out[case.name + "_Y"] = Y.t.view(torch.int16).cpu().numpy()
        if "dX" in bufs:
            dXr, dAr, dBr = olin.lora_linear_bwd(Wd, f64(d["X"]), f64(d["dY"]), f64(d["A"]), f64(d["B"]), d["s"])
            for name, ref in (("dX", dXr), ("dA", dAr), ("dB", dBr)):
                assert _rel(f64(bufs[name].t), ref) <= TOL, (case.name, name)
            out[case.name + "_dX"] = bufs["dX"].t.view(torch.int16).cpu().numpy()


def run_all() -> dict:
    q.load()
    out = {}
    _quant_cases(out)
    _linear_cases(out)
    return out


if __name__ == "__main__":
    res = run_all()
    np.savez(sys.argv[1], library=np.array(os.path.basename(q.loaded_path() or "")), **res)
    print("canary cases ok:", q.loaded_path())
