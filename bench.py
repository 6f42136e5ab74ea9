"""Benchmark of the QLoRA linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = forward + backward of the three LLaMA-7B-shaped NF4+LoRA projections
(q 4096x4096, up 11008x4096, down 4096x11008; 4096 tokens = batch 4 x seq 1024;
r = 64, alpha = 16) through the C-ABI library, with every input resident in HBM.
The weights are quantized once before timing (the base is quantized once up
front).  Prints ONE JSON line (rank 0).  Secondary measurements in the same
line: the standalone NF4 dequantizer (GB/s), the quantizer (GB/s) and the
few-token forward (GB/s).

Multi-GPU (torchrun): every rank runs an independent replica of the same
per-GPU work (the path has no exchange step; weak scaling), value = all
ranks' flops / the slowest rank's time.

--impl reference times the CPU oracle (the plain restatement of the method
that the tests compare against) on a bounded sample of the same workload on the
host cores, on rank 0 only.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import qlora_inputs as qi  # noqa: E402

METRIC = "QLoRA linear fwd+bwd TFLOP/s (% BF16 peak); NF4 dequant GB/s (% HBM)"
WORKLOAD = "llama7b_projections_q4096x4096_up11008x4096_down4096x11008_m4096_r64_fwd_bwd"


def peaks():
    """Roofline denominators: the measured HBM copy bandwidth and cuBLAS bf16
    GEMM rate measured on B200s of this kind (burst: a kernel timed alone, at the full
    clock; sustained: seconds of back-to-back GEMMs under the power cap, at the
    median clock recorded with it), else the recipe's fallback figures."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return {"hbm": float(p["hbm_gbs"]), "bf16": float(p["bf16_tflops"]),
                "bf16_sus": float(p["bf16_tflops_sustained"]), "src": "measured",
                "burst_mhz": float(p.get("sm_max_mhz", 1965.0)),
                "sus_mhz": float(p.get("clocks_under_load", {}).get("sm_mhz_median", 0.0)) or None}
    except Exception:
        return {"hbm": 6650.0, "bf16": 1590.0, "bf16_sus": 1400.0, "src": "fallback", "burst_mhz": 1965.0,
                "sus_mhz": 1300.0}


def traffic_record(kernel: str):
    """DRAM bytes per launch of a kernel from the committed ncu summary, if any."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) >= 2 and parts[0] == kernel:
            try:
                return float(parts[1])
            except ValueError:
                return None
    return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled every 5 ms from a background thread
    through NVML (read-only queries), so a timed region of a few tens of ms still
    gets samples; start() returns once the first sample is in.  Falls back to
    nvidia-smi polling when NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, dev: int):
        self.proc = None
        self.thread = None
        self.samples = []
        try:
            uuid = str(torch.cuda.get_device_properties(dev).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = None

    def _nvml_loop(self, nv, h, first):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_flag.is_set():
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM), int(get_reasons(h))))
            except Exception:
                pass
            first.set()
            self.stop_flag.wait(0.005)

    def start(self):
        import threading
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByUUID(self.sel) if self.sel else nv.nvmlDeviceGetHandleByIndex(0)
            self.stop_flag = threading.Event()
            first = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h, first), daemon=True)
            self.thread.start()
            first.wait(2.0)
            return
        except Exception:
            self.thread = None
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        cmd = ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.sel:
            cmd += ["-i", self.sel]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(2.0)
            rows = self.samples
            if not rows:
                return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
            reasons = sorted({name for _, _, bits in rows for name, bit in self.REASONS if bits & bit})
            return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                    "reasons": reasons, "samples": len(rows), "source": "nvml, 5 ms"}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out = ""
        rows = [ln.split(",") for ln in out.strip().splitlines() if ln.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i] and "Not" not in r[5 + i]})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "source": "nvidia-smi, 100 ms"}


# --------------------------------------------------------------------------- our arm
class Replica:
    """Device-resident inputs, outputs and workspaces of the three projections."""

    def __init__(self, q, dev, cases=qi.LLAMA7B, dq=0):
        self.q = q
        self.cases = []
        for case in cases:
            d = qi.make_linear(case)
            w = q.quantize_nf4(d["W"].to(dev), dq=dq)
            M, N, K, r = case.M, case.N, case.K, case.r
            c = {"case": case, "w": w, "s": case.s,
                 "X": d["X"].to(dev), "A": d["A"].to(dev), "B": d["B"].to(dev), "dY": d["dY"].to(dev),
                 "Y": torch.empty((M, N), dtype=torch.bfloat16, device=dev),
                 "H": torch.empty((M, r), dtype=torch.float32, device=dev),
                 "dX": torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                 "dA": torch.empty((r, K), dtype=torch.float32, device=dev),
                 "dB": torch.empty((N, r), dtype=torch.float32, device=dev),
                 "wsf": torch.empty(q.workspace_bytes(q.QLORA_OP_FWD, M, N, K, r), dtype=torch.uint8, device=dev),
                 "wsb": torch.empty(q.workspace_bytes(q.QLORA_OP_BWD, M, N, K, r), dtype=torch.uint8, device=dev)}
            self.cases.append(c)
        torch.cuda.synchronize()
        assert q.device_status() == 0

    def flops(self):
        return sum(c["case"].flops_fwd_bwd() for c in self.cases)

    def gemm_flops(self):
        """Algorithmic flops of the fused dequant-GEMM launches of one step."""
        tot = 0
        for c in self.cases:
            M, N, K, r = c["case"].M, c["case"].N, c["case"].K, c["case"].r
            tot += (2 * M * N * K + 2 * M * r * N) + (2 * M * N * K + 2 * M * r * K)
        return tot

    def step(self):
        q = self.q
        for c in self.cases:
            q.linear_fwd(c["w"], c["X"], c["A"], c["B"], c["s"], out=c["Y"], h_out=c["H"], workspace=c["wsf"])
            q.linear_bwd(c["w"], c["X"], c["dY"], c["A"], c["B"], c["s"], H=c["H"],
                         outs=(c["dX"], c["dA"], c["dB"]), workspace=c["wsb"])


def timed(fn, steps, barrier):
    barrier()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    barrier()
    return a.elapsed_time(b)


def run_ours(args, rank, world, dev, barrier, allmax):
    import bit_quantized_lora_nf4_b200 as q
    q.load()
    pk = peaks()
    rep = Replica(q, dev)
    for _ in range(args.warmup):
        rep.step()
    torch.cuda.synchronize()

    clk = ClockSampler(dev)
    clk.start()
    ms = timed(rep.step, args.steps, barrier)
    clocks = clk.stop()
    assert q.device_status() == 0
    ms_max = allmax(ms)
    ms_step = ms_max / args.steps
    value = whole_job_rate(world, rep.flops(), ms_step) / 1e12

    # kernel-level roofline pass: the library records events around its own launches
    kp = min(args.steps, 50)
    q.profile_enable(True)
    timed(rep.step, kp, barrier)
    g_fwd_ms, g_fwd_n = q.profile_read(q.PROF_GEMM_FWD)
    g_dg_ms, g_dg_n = q.profile_read(q.PROF_GEMM_DGRAD)
    lora_ms, lora_n = q.profile_read(q.PROF_LORA)
    all_ms, all_n = q.profile_read(q.PROF_ALL)
    q.profile_enable(False)
    gemm_ms = (g_fwd_ms + g_dg_ms) / kp
    launches_per_gemm = (g_fwd_n + g_dg_n) / kp
    achieved = rep.gemm_flops() / (gemm_ms * 1e-3) / 1e12
    per_launch_flops = rep.gemm_flops() / launches_per_gemm
    # The GEMM launches are timed inside a region of a few tens of ms at the clock the
    # sampler records, so the burst peak (a GEMM timed alone at the full clock) is the
    # matching denominator; the sustained one (seconds under the power cap, at a lower
    # median clock) is kept beside it.
    roofline = {"bound": "tensor", "kernel": "qgemm2_kernel (fused NF4 dequant-GEMM, forward + dgrad)",
                "achieved": round(achieved, 1), "peak": pk["bf16"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16"], 4),
                "peak_kind": f"bf16 dense, burst ({pk['src']}, at {pk['burst_mhz']:.0f} MHz); "
                             f"timed region median SM clock {clocks.get('sm_mhz')} MHz",
                "frac_of_sustained_peak": round(achieved / pk["bf16_sus"], 4),
                "sustained_peak": pk["bf16_sus"], "sustained_peak_mhz": pk["sus_mhz"],
                "flops_per_launch": per_launch_flops,
                "traffic": traffic_record("qgemm2_kernel"),
                "share_of_step": round(gemm_ms / (all_ms / kp), 3),
                "adapter_gemms_ms_per_step": round(lora_ms / kp, 4)}
    gpu_launches = int(round(all_n / kp * args.steps))

    extras = measure_extras(q, rep, dev, pk, barrier)
    extras["llama65b"] = measure_65b(q, dev, pk, barrier)
    extras["decoder_layer"] = measure_layer(q, dev, pk, barrier)
    extras["dq_signed"] = measure_dq_signed(q, dev, pk, barrier)
    extras["lq_decompose"] = measure_lq(q, dev, pk, barrier)
    extras["dense_base"] = measure_dense(q, rep, dev, pk, barrier)
    e2e = measure_e2e(q, rep, dev, min(args.steps, 20), barrier, allmax, world)

    line = {"metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "tokens": 4096, "r": 64, "alpha": 16,
                       "flops_per_step_per_gpu": rep.flops(),
                       "l2": "inputs larger than L2 (about 620 MB of activations, gradients and outputs per step)",
                       "parallelism": f"replicas x{world}"},
            "frac_of_bf16_peak": round(value / world / pk["bf16"], 4),
            "roofline": roofline, "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clocks}
    line.update(extras)
    if rank == 0:
        line["cpu_baseline"] = cpu_baseline(world)
        print(json.dumps(line), flush=True)


def measure_layer(q, dev, pk, barrier):
    """One fwd + bwd step of a LLaMA-7B-shaped decoder layer (batch 4 x seq 2048, d 4096, 32 heads,
    SwiGLU 11008, RMSNorm) whose seven projections are the library's NF4 + LoRA (r = 64) linears and
    whose glue (norms, rotary embedding, attention, SwiGLU) is torch.  The linears' share is measured
    by the library's own per-launch events in a second pass."""
    import qlora_layer as ql
    cfg = ql.LayerConfig()
    params = ql.make_params(cfg, seed=21)
    layer = ql.QLoRADecoderLayer(cfg, params, dev)
    del params
    g = torch.Generator(device=dev).manual_seed(3)
    x = torch.randn(4, 2048, cfg.d, generator=g, device=dev).to(torch.bfloat16)
    gout = torch.randn(4, 2048, cfg.d, generator=g, device=dev).to(torch.bfloat16)

    def step():
        for _, A, B in layer.adapters():
            A.grad = None
            B.grad = None
        xd = x.detach().requires_grad_(True)
        out = layer(xd)
        (out.float() * gout.float()).sum().backward()
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    steps = 10
    ms = timed(step, steps, barrier) / steps
    q.profile_enable(True)
    for _ in range(5):
        step()
    torch.cuda.synchronize()
    lib_ms, _ = q.profile_read(q.PROF_ALL)
    q.profile_enable(False)
    lib_ms /= 5
    flops = cfg.linear_flops_fwd_bwd(4 * 2048)
    tf = flops / (lib_ms * 1e-3) / 1e12
    out = {"ms_per_step": round(ms, 3), "linear_ms_per_step": round(lib_ms, 3),
           "linear_tflops": round(tf, 1), "linear_frac_of_bf16_peak": round(tf / pk["bf16"], 4),
           "linear_frac_of_sustained_peak": round(tf / pk["bf16_sus"], 4),
           "linear_flops_per_step": flops, "step_tflops_counting_linears": round(flops / (ms * 1e-3) / 1e12, 1),
           "workload": "llama7b_decoder_layer_b4_s2048_d4096_h32_ffn11008_r64_fwd_bwd_7_nf4_lora_linears"}
    del layer, x, gout
    torch.cuda.empty_cache()
    return out


def measure_65b(q, dev, pk, barrier):
    """The LLaMA-65B-shaped projections (8192 x 8192, 22016 x 8192, 8192 x 22016; 8192 tokens, r = 64),
    one fwd + bwd of each per step, device-timed like the main line (a parity-test configuration,
    reported beside the main line)."""
    rep = Replica(q, dev, qi.LLAMA65B)
    for _ in range(3):
        rep.step()
    torch.cuda.synchronize()
    steps = 10
    ms = timed(rep.step, steps, barrier) / steps
    tf = rep.flops() / (ms * 1e-3) / 1e12
    out = {"value": round(tf, 1), "unit": "TFLOP/s", "ms_per_step": round(ms, 3),
           "frac_of_bf16_peak": round(tf / pk["bf16"], 4),
           "frac_of_sustained_peak": round(tf / pk["bf16_sus"], 4), "flops_per_step": rep.flops(),
           "workload": "llama65b_projections_q8192x8192_up22016x8192_down8192x22016_m8192_r64_fwd_bwd"}
    del rep
    torch.cuda.empty_cache()
    return out


def dequant_gbs(q, cases, dev, pk, barrier):
    """Standalone dequantizer over the cases' weights: 0.5 + 1/64 + 4/16384 B in, 2 B out per weight."""
    bufs = [torch.empty((c["case"].N, c["case"].K), dtype=torch.bfloat16, device=dev) for c in cases]
    nw = sum(c["case"].N * c["case"].K for c in cases)
    dq_bytes = sum(c["w"].nbytes() for c in cases) + 2 * nw

    def dq():
        for c, b in zip(cases, bufs):
            q.dequantize(c["w"], out=b)
    # ten warm-up rounds: the first calls after the fwd + bwd step also write back the step's dirty
    # outputs from L2 (about 126 MB), which is not the dequantizer's traffic
    for _ in range(10):
        dq()
    reps = 20
    ms = timed(dq, reps, barrier) / reps
    gbs = dq_bytes / (ms * 1e-3) / 1e9
    return {"value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / pk["hbm"], 4),
            "peak": pk["hbm"], "bytes_per_weight": round(dq_bytes / nw, 4)}


def quantize_gbs(q, cases, dev, pk, barrier, dq=0):
    """Quantizer over fresh fp32 copies of the cases' shapes: 4 B in, 0.516 B out per weight
    (the signed reading's workspace round trip of 4 B per block is not counted)."""
    nw = sum(c["case"].N * c["case"].K for c in cases)
    Ws = [torch.randn((c["case"].N, c["case"].K), device=dev, dtype=torch.float32) * 0.02 for c in cases]
    tmp = [q.NF4Weight.empty(c["case"].N, c["case"].K, dev, dq=dq) for c in cases]
    wss = [torch.empty(max(16, q.load().qlora_quantize_workspace_bytes(c["case"].N, c["case"].K, dq)),
                       dtype=torch.uint8, device=dev) for c in cases]

    def qz():
        for W, t, ws in zip(Ws, tmp, wss):
            q.quantize_nf4(W, out=t, workspace=ws)
    for _ in range(3):
        qz()
    ms = timed(qz, 10, barrier) / 10
    qb = 4 * nw + sum(t.nbytes() for t in tmp)
    gbs = qb / (ms * 1e-3) / 1e9
    del Ws, tmp, wss
    return {"value": round(gbs, 1), "unit": "GB/s", "frac": round(gbs / pk["hbm"], 4)}


def measure_dq_signed(q, dev, pk, barrier):
    """The signed reading of the block constants (int8 codes around the tensor-wide mean mu): one
    fwd + bwd step of the LLaMA-7B projections, the dequantizer and the quantizer with such weights,
    and the error of the constants and of the weight against the plain reading."""
    rep = Replica(q, dev, qi.LLAMA7B, dq=q.DQ_SIGNED)
    for _ in range(3):
        rep.step()
    torch.cuda.synchronize()
    steps = 10
    ms = timed(rep.step, steps, barrier) / steps
    tf = rep.flops() / (ms * 1e-3) / 1e12
    out = {"step": {"value": round(tf, 1), "unit": "TFLOP/s", "ms_per_step": round(ms, 4),
                    "frac_of_bf16_peak": round(tf / pk["bf16"], 4),
                    "frac_of_sustained_peak": round(tf / pk["bf16_sus"], 4)},
           "dequant": dequant_gbs(q, rep.cases, dev, pk, barrier),
           "quantize": quantize_gbs(q, rep.cases, dev, pk, barrier, dq=q.DQ_SIGNED)}
    Wq = qi.make_weight(4096, 4096, qi.LLAMA7B[0].seed).to(dev)
    a = Wq.reshape(-1, 64).abs().amax(dim=1).double()
    for name, dq in (("plain", q.DQ_PLAIN), ("signed", q.DQ_SIGNED)):
        wq = q.quantize_nf4(Wq, dq=dq)
        d = q.dequantize(wq).double() - Wq.double()
        # a' of every block from the stored bytes (fp32 products and sums, as the kernels form them)
        S = wq.scales.repeat_interleave(256)[:a.numel()]
        if dq == q.DQ_SIGNED:
            ap = (wq.absmax_q.view(torch.int8).float() * S) + wq.offset
        else:
            ap = wq.absmax_q.float() * S
        out[name] = {"weight_rel_frobenius_error": round(float(d.norm() / Wq.double().norm()), 6),
                     "block_constant_mean_abs_rel_error": round(float(((ap.double() - a).abs() / a).mean()), 6)}
        del wq, d
    out["note"] = "errors on the 4096x4096 Gaussian q-projection weight"
    out["workload"] = "llama7b_projections_m4096_r64_fwd_bwd_signed_block_constants"
    del rep, Wq
    torch.cuda.empty_cache()
    return out


TF32_OVER_BF16 = 1.1 / 2.25   # nominal dense tf32 / bf16 tensor throughput of the B200


def measure_lq(q, dev, pk, barrier):
    """Low-rank plus quantized decomposition of the 4096 x 4096 q-projection-shaped weight with a
    planted rank-64 part (r = 64, test matrix width 72, 2 power rounds, 2 alternation rounds):
    time per decomposition, and the residual products (tcgen05 tf32, three products per tile) against
    HBM (they read W and the packed weight once per launch) and against the tf32 tensor peak."""
    N = K = 4096
    r, l, power, iters = 64, 72, 2, 2
    W = qi.make_lowrank_weight(N, K, r, seed=99).to(dev)
    Om = qi.make_test_matrix(K, l, seed=100).to(dev)
    ws = torch.empty(q.load().qlora_lq_workspace_bytes(N, K, r, l, 0), dtype=torch.uint8, device=dev)

    def run():
        return q.lq_decompose(W, r, Om, power=power, iters=iters, workspace=ws)
    for _ in range(2):
        run()
    torch.cuda.synchronize()
    reps = 3
    ms = timed(run, reps, barrier) / reps
    q.profile_enable(True)
    w, L1, L2, err = run()
    torch.cuda.synchronize()
    pms, pn = q.profile_read(q.PROF_LQ_PRODUCT)
    parts = {name: round(q.profile_read(k)[0], 3) for name, k in (
        ("products", q.PROF_LQ_PRODUCT), ("residual_and_error", q.PROF_LQ_RESIDUAL), ("cholesky", q.PROF_LQ_CHOL),
        ("jacobi", q.PROF_LQ_JACOBI), ("gram_small_sums", q.PROF_LQ_SMALL), ("quantizer", q.PROF_QUANT))}
    q.profile_enable(False)
    flops = pn * 2 * N * K * l
    tf = flops / (pms * 1e-3) / 1e12
    # algorithmic bytes: the first rank-r step (6 launches) reads W alone (4 B per element), the later
    # ones (12) W and the packed weight (4 + 0.5 + 1/64 + 4/16384 B); every launch reads its l-wide
    # small operand and writes its l-wide result (4 l (N + K) bytes)
    n_plain = 6 if pn >= 6 else pn
    per_elem = n_plain * 4.0 + (pn - n_plain) * (4.0 + 0.5 + 1.0 / 64 + 4.0 / 16384)
    prod_bytes = per_elem * N * K + pn * 4.0 * l * (N + K)
    gbs = prod_bytes / (pms * 1e-3) / 1e9
    tf32_peak = pk["bf16"] * TF32_OVER_BF16
    plain = q.quantize_nf4(W)
    plain_err = float((q.dequantize(plain).double() - W.double()).norm() / W.double().norm())
    e = err.cpu().numpy()
    out = {"ms_per_decomposition": round(ms, 3),
           "products": {"launches": int(pn), "ms": round(pms, 3), "bound": "hbm", "achieved": round(gbs, 1),
                        "unit": "GB/s", "peak": pk["hbm"], "frac": round(gbs / pk["hbm"], 4),
                        "bytes_per_launch_avg": round(prod_bytes / max(pn, 1)),
                        "tflops": round(tf, 2), "tf32_peak": round(tf32_peak, 1),
                        "frac_of_tf32_peak": round(tf / tf32_peak, 4),
                        "tf32_peak_kind": "measured bf16 burst x nominal tf32/bf16 (1.1 / 2.25)",
                        "share": round(pms / ms, 3), "flops_per_launch": 2 * N * K * l},
           "ms_by_kernel_kind": parts,
           "rel_error": {"plain_nf4": round(plain_err, 5), "after_quantization": [round(x, 5) for x in e[:, 0]],
                         "after_rank_r_step": [round(x, 5) for x in e[:, 1]]},
           "workload": "lq_decompose_4096x4096_planted_rank64_r64_l72_power2_iters2"}
    del W, Om, ws, w, L1, L2, plain
    torch.cuda.empty_cache()
    return out


def measure_dense(q, rep, dev, pk, barrier):
    """The LLaMA-7B projection step (M = 4096, r = 64, fwd + bwd) on dense bf16 base weights (the
    call a weight from any quantizer takes): once with W' already materialized, once re-materializing
    it in every pass through qlora_linear_*_materialized with the library's dequantizer as the
    black box."""
    import ctypes
    lib = q.load()
    dense = [q.dequantize(c["w"]) for c in rep.cases]
    scratch = [torch.empty_like(W) for W in dense]
    wsf = [torch.empty(lib.qlora_workspace_bytes(q.QLORA_OP_FWD_DENSE, c["case"].M, c["case"].N, c["case"].K,
                                                 c["case"].r), dtype=torch.uint8, device=dev) for c in rep.cases]
    wsb = [torch.empty(lib.qlora_workspace_bytes(q.QLORA_OP_BWD_DENSE, c["case"].M, c["case"].N, c["case"].K,
                                                 c["case"].r), dtype=torch.uint8, device=dev) for c in rep.cases]
    st = lambda: ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)   # noqa: E731
    P = lambda t: ctypes.c_void_p(t.data_ptr())                              # noqa: E731
    structs = [c["w"].c_struct() for c in rep.cases]

    def mat(ctx, w_out, n, k, stream):
        i = ctx or 0          # ctypes hands a NULL context (case 0) over as None
        return lib.qlora_dequantize(ctypes.byref(structs[i]), ctypes.c_void_p(w_out), ctypes.c_void_p(stream))
    fn = q.MATERIALIZE_FN(mat)

    def step(materialize):
        for i, c in enumerate(rep.cases):
            M, N, K, r = c["case"].M, c["case"].N, c["case"].K, c["case"].r
            if materialize:
                q._check(lib.qlora_linear_fwd_materialized(fn, ctypes.c_void_p(i), P(scratch[i]), N, K, P(c["X"]), M,
                                                           P(c["A"]), P(c["B"]), r, c["s"], P(c["Y"]), P(c["H"]),
                                                           P(wsf[i]), wsf[i].numel(), st()), "fwd_materialized")
                q._check(lib.qlora_linear_bwd_materialized(fn, ctypes.c_void_p(i), P(scratch[i]), N, K, P(c["X"]),
                                                           P(c["dY"]), M, P(c["A"]), P(c["B"]), r, c["s"], P(c["H"]),
                                                           P(c["dX"]), P(c["dA"]), P(c["dB"]), P(wsb[i]),
                                                           wsb[i].numel(), st()), "bwd_materialized")
            else:
                q._check(lib.qlora_linear_fwd_dense(P(dense[i]), N, K, P(c["X"]), M, P(c["A"]), P(c["B"]), r, c["s"],
                                                    P(c["Y"]), P(c["H"]), P(wsf[i]), wsf[i].numel(), st()),
                         "fwd_dense")
                q._check(lib.qlora_linear_bwd_dense(P(dense[i]), N, K, P(c["X"]), P(c["dY"]), M, P(c["A"]),
                                                    P(c["B"]), r, c["s"], P(c["H"]), P(c["dX"]), P(c["dA"]),
                                                    P(c["dB"]), P(wsb[i]), wsb[i].numel(), st()), "bwd_dense")
    out = {}
    for name, m in (("dense_weight", False), ("materialized_each_pass", True)):
        for _ in range(3):
            step(m)
        torch.cuda.synchronize()
        ms = timed(lambda: step(m), 20, barrier) / 20
        out[name] = {"ms_per_step": round(ms, 4), "value": round(rep.flops() / (ms * 1e-3) / 1e12, 1),
                     "unit": "TFLOP/s"}
    assert q.device_status() == 0
    out["workload"] = "llama7b_projections_m4096_r64_fwd_bwd_dense_bf16_base"
    del dense, scratch, wsf, wsb
    torch.cuda.empty_cache()
    return out


def measure_extras(q, rep, dev, pk, barrier):
    """Standalone dequantizer, quantizer and few-token forward, each in GB/s."""
    out = {"dequant": dequant_gbs(q, rep.cases, dev, pk, barrier),
           "quantize": quantize_gbs(q, rep.cases, dev, pk, barrier)}
    # few-token forward: weights rotated over enough copies to exceed L2
    res = {}
    for M in qi.GEMV_TOKENS:
        tot_bytes, tot_ms = 0, 0.0
        for c in rep.cases:
            case = c["case"]
            ncopy = max(2, int(np.ceil(400e6 / c["w"].nbytes())))
            copies = [c["w"]] + [q.NF4Weight(case.N, case.K, c["w"].codes.clone(), c["w"].absmax_q.clone(),
                                             c["w"].group_scale.clone()) for _ in range(ncopy - 1)]
            X = c["X"][:M].contiguous()
            Y = torch.empty((M, case.N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty(q.workspace_bytes(q.QLORA_OP_FWD, M, case.N, case.K, case.r), dtype=torch.uint8,
                             device=dev)

            def calls():
                for w in copies:
                    q.linear_fwd(w, X, c["A"], c["B"], c["s"], save_h=False, out=Y, workspace=ws)
            # one CUDA graph holds one call per weight copy, so the timing sees the GPU,
            # not the Python/ctypes call overhead of these few-microsecond calls
            side = torch.cuda.Stream()
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                calls()
            torch.cuda.current_stream().wait_stream(side)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                calls()
            for _ in range(3):
                graph.replay()
            reps = 4
            ms = timed(graph.replay, reps, barrier) / (reps * ncopy)
            del graph
            nbytes = c["w"].nbytes() + 2 * case.r * (case.N + case.K) + 2 * M * (case.N + case.K)
            tot_bytes += nbytes
            tot_ms += ms
            del copies
        gbs = tot_bytes / (tot_ms * 1e-3) / 1e9
        res[str(M)] = {"value": round(gbs, 1), "frac": round(gbs / pk["hbm"], 4), "us_per_call_avg": round(
            1e3 * tot_ms / len(rep.cases), 2)}
    # the 4-bit tables the pages compare NF4 against: reconstruction error through the library
    Wq = qi.make_weight(4096, 4096, qi.LLAMA7B[0].seed).to(dev)
    errs, shares = {}, {}
    for name, fid in (("nf4", q.FORMAT_NF4), ("fp4", q.FORMAT_FP4), ("int4", q.FORMAT_INT4)):
        wq = q.quantize_nf4(Wq, format=fid)
        d = q.dequantize(wq).double() - Wq.double()
        errs[name] = round(float(d.norm() / Wq.double().norm()), 5)
        # how evenly the codes use the 16 levels (the pages: at normal quantiles every level
        # takes about the same share of Gaussian weights; absmax scaling makes it approximate)
        c = torch.stack([wq.codes & 15, wq.codes >> 4]).reshape(-1).long()
        h = torch.bincount(c, minlength=16).double()
        p_ = h / h.sum()
        used = p_[p_ > 0]
        shares[name] = {"code_share": [round(float(x), 5) for x in p_],
                        "entropy_bits": round(float(-(used * used.log2()).sum()), 4),
                        "max_over_min_share": round(float(used.max() / used.min()), 3)}
        del wq, d, c
    del Wq
    out["formats"] = {"rel_frobenius_error": errs, "level_use": shares,
                      "note": "||dequant(quant(W)) - W|| / ||W|| and the share of weights on each of the 16 "
                              "levels (entropy of the codes, 4 bits = equal shares) on the 4096x4096 "
                              "Gaussian q-projection weight, blocks of 64, double-quantized constants"}
    out["gemv"] = {"unit": "GB/s", "tokens": res,
                   "note": "packed weight + adapters + X + Y bytes per call; calls replayed from a CUDA graph, "
                           "weights rotated over copies totalling > 400 MB (beyond L2)"}
    return out


def measure_e2e(q, rep, dev, steps, barrier, allmax, world):
    """Same step through the C-ABI with host buffers: every step copies X and dY in from pinned host
    memory and Y, dX, dA, dB back out.  The copies run on their own streams (host-to-device and
    device-to-host use separate copy engines, and the link is full duplex) and the device buffers
    are double-buffered, so one projection's copies overlap another's compute; every byte of every
    step still crosses the link inside the timed region."""
    host = []
    for c in rep.cases:
        host.append({k: c[k].cpu().pin_memory() for k in ("X", "dY")} |
                    {k: torch.empty_like(c[k], device="cpu").pin_memory() for k in ("Y", "dX", "dA", "dB")})
    h2d = sum(h["X"].numel() * 2 + h["dY"].numel() * 2 for h in host)
    d2h = sum(h["Y"].numel() * 2 + h["dX"].numel() * 2 + h["dA"].numel() * 4 + h["dB"].numel() * 4 for h in host)
    keys_in, keys_out = ("X", "dY"), ("Y", "dX", "dA", "dB")
    # two device buffer sets per projection
    bufs = [[{k: torch.empty_like(c[k]) for k in keys_in + keys_out + ("H",)} for _ in range(2)] for c in rep.cases]
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {}

    def event(key):
        if key not in ev:
            ev[key] = torch.cuda.Event()
        return ev[key]

    state = {"u": 0}

    def unit(ci):
        c, h = rep.cases[ci], host[ci]
        u = state["u"]
        state["u"] += 1
        bset = (ci, u // len(rep.cases) % 2)
        dbuf = bufs[ci][bset[1]]
        with torch.cuda.stream(s_in):        # inputs may be overwritten once the compute that read them is done
            if ("comp", bset) in ev:
                s_in.wait_event(ev[("comp", bset)])
            for k in keys_in:
                dbuf[k].copy_(h[k], non_blocking=True)
            event(("in", bset)).record(s_in)
        comp.wait_event(ev[("in", bset)])
        if ("out", bset) in ev:              # outputs may be overwritten once they are copied out
            comp.wait_event(ev[("out", bset)])
        q.linear_fwd(c["w"], dbuf["X"], c["A"], c["B"], c["s"], out=dbuf["Y"], h_out=dbuf["H"], workspace=c["wsf"])
        q.linear_bwd(c["w"], dbuf["X"], dbuf["dY"], c["A"], c["B"], c["s"], H=dbuf["H"],
                     outs=(dbuf["dX"], dbuf["dA"], dbuf["dB"]), workspace=c["wsb"])
        event(("comp", bset)).record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev[("comp", bset)])
            for k in keys_out:
                h[k].copy_(dbuf[k], non_blocking=True)
            event(("out", bset)).record(s_out)

    def st():
        for ci in range(len(rep.cases)):
            unit(ci)

    def run(n):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        start.record(comp)
        s_in.wait_stream(comp)
        s_out.wait_stream(comp)
        for _ in range(n):
            st()
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)               # the last outputs are on the host
        end.record(comp)
        torch.cuda.synchronize()
        barrier()
        return start.elapsed_time(end)
    run(2)
    ms = allmax(run(steps)) / steps
    # the pipeline computes what the plain step computes
    for c, h in zip(rep.cases, host):
        q.linear_fwd(c["w"], c["X"], c["A"], c["B"], c["s"], out=c["Y"], h_out=c["H"], workspace=c["wsf"])
    torch.cuda.synchronize()
    for c, h in zip(rep.cases, host):
        assert torch.equal(h["Y"].to(dev), c["Y"]), "end-to-end pipeline output differs from the device step"
    return {"value": round(world * rep.flops() / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 4),
            "note": "inputs copied in and outputs copied out every step (pinned host memory); copies on "
                    "their own streams, device buffers double-buffered"}


# --------------------------------------------------------------------------- oracle (CPU) arm
def oracle_sample(Ms: int, Ns: int):
    """One bounded sample of the workload on the oracle: dequantize an Ns x 4096
    slice of the q-projection weight and run fwd + bwd for Ms tokens."""
    from oracle import linear as olin
    from oracle import nf4 as onf4
    case = qi.LLAMA7B[0]
    d = qi.make_linear(case)
    W = d["W"][:Ns].numpy()
    oq = onf4.quantize_nf4(W)                           # once, up front (not timed)
    X = d["X"][:Ms].float().numpy().astype(np.float64)
    dY = d["dY"][:Ms, :Ns].float().numpy().astype(np.float64)
    A = d["A"].float().numpy().astype(np.float64)
    B = d["B"][:Ns].float().numpy().astype(np.float64)
    flops = 4 * Ms * Ns * case.K + 6 * Ms * case.r * (case.K + Ns)

    def step():
        Wd = onf4.bf16_bits_to_f32(onf4.dequantize_nf4(oq)).astype(np.float64)
        olin.lora_linear_fwd(Wd, X, A, B, case.s)
        olin.lora_linear_bwd(Wd, X, dY, A, B, case.s)
    return step, flops


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(world):
    Ms, Ns = 1024, 1024
    step, flops = oracle_sample(Ms, Ns)
    step()
    t0 = time.perf_counter()
    n = 0
    while time.perf_counter() - t0 < 10.0 or n < 2:
        step()
        n += 1
    dt = (time.perf_counter() - t0) / n
    return {"value": round(flops / dt / 1e12, 5), "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"q-projection slice: dequantize 1024x4096 NF4 rows + fp64 fwd+bwd for 1024 tokens, "
                      f"{n} reps, {dt:.2f} s each"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    # size the per-step sample so that warmup + steps finish in about two minutes
    step, flops = oracle_sample(128, 128)
    t0 = time.perf_counter()
    step()
    t_small = time.perf_counter() - t0
    budget = 120.0 / max(1, args.steps + args.warmup)
    side = int(np.clip(128 * np.sqrt(budget / max(t_small, 1e-6)), 32, 4096)) // 16 * 16
    step, flops = oracle_sample(side, side)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    v = round(flops / dt / 1e12, 6)
    print(json.dumps({"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
                      "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3),
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "config": {"workload": WORKLOAD, "tokens": 4096, "r": 64, "alpha": 16},
                      "cpu_baseline": {"value": v, "unit": "TFLOP/s", "kind": "oracle", "cores": cpu_threads(),
                                       "sample": f"q-projection slice {side}x4096 dequantized + fp64 fwd+bwd "
                                                 f"for {side} tokens per step"},
                      "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}),
          flush=True)


# --------------------------------------------------------------------------- profiling entry
def run_ncu_case(args):
    """A small, fixed launch sequence for ncu: one projection of the LLaMA-7B
    set (inputs above L2 size for 'up' and 'down'), warmup + steps repetitions."""
    import bit_quantized_lora_nf4_b200 as q
    q.load()
    dev = torch.device("cuda", 0)
    name = args.ncu_case
    if name == "step":   # the timed step: the three projections, forward and backward
        rep = Replica(q, dev)
        for _ in range(args.warmup + args.steps):
            rep.step()
        torch.cuda.synchronize()
        assert q.device_status() == 0
        return
    if name == "quant_signed":   # the quantizer with signed block constants, up-projection weight
        case = qi.LLAMA7B[1]
        W = qi.make_weight(case.N, case.K, case.seed).to(dev)
        out = q.NF4Weight.empty(case.N, case.K, dev, dq=q.DQ_SIGNED)
        for _ in range(args.warmup + args.steps):
            q.quantize_nf4(W, out=out)
        torch.cuda.synchronize()
        assert q.device_status() == 0
        return
    if name == "lq":     # the low-rank plus quantized decomposition of a 4096 x 4096 weight
        W = qi.make_lowrank_weight(4096, 4096, 64, seed=99).to(dev)
        Om = qi.make_test_matrix(4096, 72, seed=100).to(dev)
        for _ in range(args.warmup + args.steps):
            q.lq_decompose(W, 64, Om, power=1, iters=1)
        torch.cuda.synchronize()
        assert q.device_status() == 0
        return
    case = {"q": qi.LLAMA7B[0], "up": qi.LLAMA7B[1], "down": qi.LLAMA7B[2]}.get(name, qi.LLAMA7B[1])
    M = {"gemv1": 1, "gemv16": 16}.get(name, case.M)
    d = qi.make_linear(case, M=M)
    w = q.quantize_nf4(d["W"].to(dev))
    X, A, B, dY = (d[k].to(dev) for k in ("X", "A", "B", "dY"))
    out = torch.empty((case.N, case.K), dtype=torch.bfloat16, device=dev) if name == "dequant" else None
    for _ in range(args.warmup + args.steps):
        if name == "dequant":
            q.dequantize(w, out=out)
        elif name.startswith("gemv"):
            q.linear_fwd(w, X, A, B, case.s, save_h=False)
        else:
            _, H = q.linear_fwd(w, X, A, B, case.s)
            q.linear_bwd(w, X, dY, A, B, case.s, H=H)
    torch.cuda.synchronize()
    assert q.device_status() == 0


# --------------------------------------------------------------------------- ranks
def make_comm(world: int, dev, backend: str = "nccl"):
    """(barrier, allmax, dist module or None) for one process per GPU.  Replicas only:
    the ranks share no data-path collective, only the barriers around the timed region
    and the max over ranks of its duration.  Short process-group timeout, so that ranks
    waiting for a rank that died end with an error instead of hanging."""
    if world <= 1:
        return (lambda: None), (lambda x: x), None
    import datetime
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))

    def barrier():
        dist.barrier()

    def allmax(x):
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())
    return barrier, allmax, dist


def whole_job_rate(world: int, units_per_rank: float, max_ms: float) -> float:
    """Units per second of all ranks together: every rank processes units_per_rank in
    the timed region, whose length is the slowest rank's (max over ranks)."""
    return world * units_per_rank / (max_ms * 1e-3)


# --------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ncu-case", choices=["step", "q", "up", "down", "gemv1", "gemv16", "dequant", "lq", "quant_signed"], default=None,
                    help="profiling entry: run only one projection's calls (--warmup + --steps times), no JSON")
    args = ap.parse_args()
    if args.ncu_case:
        run_ncu_case(args)
        return
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    barrier, allmax, dist = make_comm(world, dev, "nccl")
    try:
        run_ours(args, rank, world, dev, barrier, allmax)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
