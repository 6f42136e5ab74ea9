"""Thin Python binding of libqlora.so (NF4 + double quantization + LoRA linear, sm_100a).

Argument marshalling only: every step of the computation runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (device memory and streams come
from PyTorch); each call enqueues on ``torch.cuda.current_stream()``.

The library must be built (``python -m bit_quantized_lora_nf4_b200.build``);
there is no fallback: a missing or unloadable library raises at first use.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora.so")
# The debug build: the same library with the kernels' global-memory indices
# checked against their buffers (a miss latches QLORA_ERR_BOUNDS, no trap).
# QLORA_DEBUG_BOUNDS=1 in the environment makes load() pick it.
DEBUG_LIB_PATH = os.path.join(_HERE, "libqlora_debug.so")

QLORA_OP_FWD = 0
QLORA_OP_BWD = 1
QLORA_OP_FWD_DENSE = 2      # the linear on a dense bf16 base weight (any quantizer's output)
QLORA_OP_BWD_DENSE = 3
# Stream-K split of the fused GEMM's last partial wave (qlora_set_stream_k).
STREAM_K_OFF, STREAM_K_AUTO, STREAM_K_ALWAYS = 0, 1, 2

STATUS_NAMES = {
    0: "QLORA_OK", 1: "QLORA_ERR_INVALID_ARG", 2: "QLORA_ERR_UNSUPPORTED_SHAPE", 3: "QLORA_ERR_MISALIGNED",
    4: "QLORA_ERR_NONFINITE", 5: "QLORA_ERR_DEVICE_TIMEOUT", 6: "QLORA_ERR_CUDA", 7: "QLORA_ERR_WORKSPACE",
    8: "QLORA_ERR_BOUNDS",
}

# Every symbol include/qlora.h declares.
EXPORTS = (
    "qlora_codes_bytes", "qlora_absmax_bytes", "qlora_group_scale_bytes", "qlora_quantize_nf4", "qlora_dequantize",
    "qlora_workspace_bytes", "qlora_workspace_min_bytes", "qlora_set_stream_k", "qlora_linear_fwd", "qlora_linear_bwd", "qlora_nf4_codebook", "qlora_device_status",
    "qlora_status_string", "qlora_set_wait_limit", "qlora_selftest_wait_timeout", "qlora_profile_enable",
    "qlora_profile_read", "qlora_linear_fwd_noalloc", "qlora_format_codebook", "qlora_group_scale_bytes_dq",
    "qlora_quantize_workspace_bytes", "qlora_quantize_nf4_ws", "qlora_lq_workspace_bytes", "qlora_lq_decompose",
    "qlora_lq_quantize_residual", "qlora_lq_lowrank", "qlora_linear_fwd_dense", "qlora_linear_bwd_dense",
    "qlora_linear_fwd_materialized", "qlora_linear_bwd_materialized",
)

# 4-bit code tables (QLORA_FORMAT_*): NF4 is the method's type; FP4 (e2m1) and
# INT4 are the plain float and integer types it is compared against.
FORMAT_NF4, FORMAT_FP4, FORMAT_INT4 = 0, 1, 2

# Readings of the 8-bit block constants (QLORA_DQ_*): unsigned with no offset,
# or signed around the tensor-wide mean constant (stored after the group scales).
DQ_PLAIN, DQ_SIGNED = 0, 1
# size of the library-owned scratch array of qlora_linear_fwd_noalloc (include/qlora.h)
QLORA_STATIC_SCRATCH_BYTES = 8 << 20
# element types the quantizer accepts (QLORA_DTYPE_F32 / QLORA_DTYPE_BF16)
DTYPE_F32, DTYPE_BF16 = 0, 1
_WEIGHT_DTYPES = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16}

# Kernel kinds of the timing hook (qlora_profile_read).
(PROF_ALL, PROF_GEMM_FWD, PROF_GEMM_DGRAD, PROF_LORA, PROF_QUANT, PROF_DEQUANT, PROF_GEMV, PROF_LQ_PRODUCT,
 PROF_LQ_RESIDUAL, PROF_LQ_CHOL, PROF_LQ_JACOBI, PROF_LQ_SMALL) = range(12)


class QloraError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")
        self.code = code


class Nf4WeightC(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("absmax_q", ctypes.c_void_p), ("group_scale", ctypes.c_void_p), ("format", ctypes.c_int32),
                ("dq", ctypes.c_int32)]


_lib = None

# qlora_materialize_fn: (ctx, W_out, N, K, stream) -> status
MATERIALIZE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                  ctypes.c_void_p)


_lib_path = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load the library once (libqlora.so, or libqlora_debug.so when
    QLORA_DEBUG_BOUNDS=1) and declare the C signatures."""
    global _lib, _lib_path
    if _lib is not None:
        return _lib
    if path is None:
        path = DEBUG_LIB_PATH if os.environ.get("QLORA_DEBUG_BOUNDS") == "1" else LIB_PATH
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built at {path}; run python -m bit_quantized_lora_nf4_b200.build")
    lib = ctypes.CDLL(path)
    _lib_path = path
    vp, i64, sz, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int, ctypes.c_float
    wp = ctypes.POINTER(Nf4WeightC)
    sig = {
        "qlora_codes_bytes": (sz, [i64, i64]),
        "qlora_absmax_bytes": (sz, [i64, i64]),
        "qlora_group_scale_bytes": (sz, [i64, i64]),
        "qlora_quantize_nf4": (i32, [vp, i32, wp, vp]),
        "qlora_dequantize": (i32, [wp, vp, vp]),
        "qlora_workspace_bytes": (sz, [i32, i64, i64, i64, i32]),
        "qlora_workspace_min_bytes": (sz, [i32, i64, i64, i64, i32]),
        "qlora_set_stream_k": (i32, [i32]),
        "qlora_linear_fwd": (i32, [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_bwd": (i32, [wp, vp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]),
        "qlora_nf4_codebook": (i32, [ctypes.POINTER(ctypes.c_float)]),
        "qlora_format_codebook": (i32, [i32, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float)]),
        "qlora_device_status": (i32, [vp]),
        "qlora_status_string": (ctypes.c_char_p, [i32]),
        "qlora_set_wait_limit": (ctypes.c_uint64, [ctypes.c_uint64]),
        "qlora_selftest_wait_timeout": (i32, [ctypes.c_uint64, vp]),
        "qlora_profile_enable": (None, [i32]),
        "qlora_profile_read": (i32, [i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)]),
        "qlora_linear_fwd_noalloc": (i32, [wp, vp, i64, vp, vp, i32, f32, vp, vp, vp]),
        "qlora_group_scale_bytes_dq": (sz, [i64, i64, i32]),
        "qlora_quantize_workspace_bytes": (sz, [i64, i64, i32]),
        "qlora_quantize_nf4_ws": (i32, [vp, i32, wp, vp, sz, vp]),
        "qlora_lq_workspace_bytes": (sz, [i64, i64, i32, i32, i32]),
        "qlora_lq_decompose": (i32, [vp, wp, vp, vp, i32, vp, i32, i32, i32, vp, vp, sz, vp]),
        "qlora_lq_quantize_residual": (i32, [vp, vp, vp, i32, wp, vp, sz, vp]),
        "qlora_lq_lowrank": (i32, [vp, i64, i64, wp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
        "qlora_linear_fwd_dense": (i32, [vp, i64, i64, vp, i64, vp, vp, i32, f32, vp, vp, vp, sz, vp]),
        "qlora_linear_bwd_dense": (i32, [vp, i64, i64, vp, vp, i64, vp, vp, i32, f32, vp, vp, vp, vp, vp, sz, vp]),
        "qlora_linear_fwd_materialized": (i32, [MATERIALIZE_FN, vp, vp, i64, i64, vp, i64, vp, vp, i32, f32, vp, vp,
                                                vp, sz, vp]),
        "qlora_linear_bwd_materialized": (i32, [MATERIALIZE_FN, vp, vp, i64, i64, vp, vp, i64, vp, vp, i32, f32, vp,
                                                vp, vp, vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def loaded_path() -> str | None:
    """Path of the library load() opened (None before the first load)."""
    return _lib_path


def _check(code: int, where: str):
    if code != 0:
        raise QloraError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@dataclass
class NF4Weight:
    """Frozen base weight [rows, cols] in NF4 with double-quantized constants (device tensors)."""
    rows: int
    cols: int
    codes: torch.Tensor        # uint8 [ceil(rows*cols/2)]
    absmax_q: torch.Tensor     # uint8 [ceil(rows*cols/64)] (int8 bit patterns for DQ_SIGNED)
    group_scale: torch.Tensor  # float32 [ceil(rows*cols/16384)] (+ mu last for DQ_SIGNED)
    format: int = FORMAT_NF4   # code table (FORMAT_*)
    dq: int = DQ_PLAIN         # reading of the block constants (DQ_*)

    def c_struct(self) -> Nf4WeightC:
        return Nf4WeightC(self.rows, self.cols, self.codes.data_ptr(), self.absmax_q.data_ptr(),
                          self.group_scale.data_ptr(), self.format, self.dq)

    @staticmethod
    def empty(rows: int, cols: int, device="cuda", format: int = FORMAT_NF4, dq: int = DQ_PLAIN) -> "NF4Weight":
        lib = load()
        gs = lib.qlora_group_scale_bytes_dq(rows, cols, dq)
        if gs == 0:
            raise QloraError(1, "NF4Weight.empty")
        return NF4Weight(rows, cols,
                         torch.empty(lib.qlora_codes_bytes(rows, cols), dtype=torch.uint8, device=device),
                         torch.empty(lib.qlora_absmax_bytes(rows, cols), dtype=torch.uint8, device=device),
                         torch.empty(gs // 4, dtype=torch.float32, device=device), format, dq)

    @property
    def scales(self) -> torch.Tensor:
        """The per-group scales S_g (without the offset)."""
        return self.group_scale[:-1] if self.dq == DQ_SIGNED else self.group_scale

    @property
    def offset(self) -> torch.Tensor | None:
        """mu, the offset of DQ_SIGNED block constants (a 1-element view), else None."""
        return self.group_scale[-1:] if self.dq == DQ_SIGNED else None

    def nbytes(self) -> int:
        return self.codes.numel() + self.absmax_q.numel() + 4 * self.group_scale.numel()


def codebook(format: int = FORMAT_NF4, thresholds: bool = False):
    """The 16 levels of a code table (and its 15 decision thresholds when asked)."""
    lib = load()
    lv = (ctypes.c_float * 16)()
    th = (ctypes.c_float * 15)()
    _check(lib.qlora_format_codebook(format, lv, th), "qlora_format_codebook")
    return (list(lv), list(th)) if thresholds else list(lv)


def workspace_bytes(op: int, M: int, N: int, K: int, r: int) -> int:
    return int(load().qlora_workspace_bytes(op, M, N, K, r))


def device_status() -> int:
    return int(load().qlora_device_status(_stream()))


def set_wait_limit(cycles: int) -> int:
    return int(load().qlora_set_wait_limit(cycles))


def set_stream_k(mode: int) -> int:
    """STREAM_K_OFF / _AUTO (default) / _ALWAYS; returns the previous mode."""
    prev = int(load().qlora_set_stream_k(mode))
    if prev < 0:
        raise ValueError(f"unknown stream-K mode {mode}")
    return prev


def selftest_wait_timeout(cycles: int) -> int:
    lib = load()
    _check(lib.qlora_selftest_wait_timeout(cycles, _stream()), "qlora_selftest_wait_timeout")
    return device_status()


def profile_enable(on: bool) -> None:
    load().qlora_profile_enable(1 if on else 0)


def profile_read(kind: int):
    """(summed kernel time in ms, launch count) of one kernel kind since profile_enable(True)."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(load().qlora_profile_read(kind, ctypes.byref(ms), ctypes.byref(n)), "qlora_profile_read")
    return ms.value, n.value


def quantize_nf4(W: torch.Tensor, out: NF4Weight | None = None, format: int = FORMAT_NF4,
                 dq: int = DQ_PLAIN, workspace: torch.Tensor | None = None) -> NF4Weight:
    """Quantize a contiguous fp32 or bf16 CUDA tensor [rows, cols] (flat
    row-major) to a 4-bit table (NF4 unless `format` says otherwise) with block
    constants as `dq` reads them (`out.format` / `out.dq` when `out` is given).
    DQ_SIGNED uses a workspace of qlora_quantize_workspace_bytes (allocated here
    when not given)."""
    lib = load()
    assert W.is_cuda and W.dtype in _WEIGHT_DTYPES and W.is_contiguous()
    rows, cols = (W.shape[0], W[0].numel()) if W.dim() >= 2 else (1, W.numel())
    w = out if out is not None else NF4Weight.empty(rows, cols, W.device, format, dq)
    s = w.c_struct()
    need = int(lib.qlora_quantize_workspace_bytes(rows, cols, w.dq))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.qlora_quantize_nf4_ws(_ptr(W), _WEIGHT_DTYPES[W.dtype], ctypes.byref(s), _ptr(workspace), nbytes,
                                     _stream()),
           "qlora_quantize_nf4_ws")
    return w


def lq_decompose(W: torch.Tensor, r: int, Omega: torch.Tensor, power: int = 2, iters: int = 4,
                 format: int = FORMAT_NF4, dq: int = DQ_PLAIN, workspace: torch.Tensor | None = None):
    """W ~ W'(Q) + L1 L2 (qlora_lq_decompose).  W: contiguous fp32 CUDA [N, K];
    Omega: fp32 CUDA [K, l] test matrix.  Returns (NF4Weight Q, L1 fp32 [N, r],
    L2 fp32 [r, K], err fp64 [iters, 2]: relative error after each round's
    quantization and after its rank-r step)."""
    lib = load()
    assert W.is_cuda and W.dtype == torch.float32 and W.is_contiguous() and W.dim() == 2
    assert Omega.is_cuda and Omega.dtype == torch.float32 and Omega.is_contiguous()
    N, K = W.shape
    l = Omega.shape[1]
    w = NF4Weight.empty(N, K, W.device, format, dq)
    L1 = torch.empty((N, r), dtype=torch.float32, device=W.device)
    L2 = torch.empty((r, K), dtype=torch.float32, device=W.device)
    err = torch.empty((iters, 2), dtype=torch.float64, device=W.device)
    need = int(lib.qlora_lq_workspace_bytes(N, K, r, l, dq))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=W.device)
    s = w.c_struct()
    _check(lib.qlora_lq_decompose(_ptr(W), ctypes.byref(s), _ptr(L1), _ptr(L2), r, _ptr(Omega), l, power, iters,
                                  _ptr(err), _ptr(workspace), workspace.numel(), _stream()), "qlora_lq_decompose")
    return w, L1, L2, err


def lq_quantize_residual(W: torch.Tensor, L1: torch.Tensor, L2: torch.Tensor, format: int = FORMAT_NF4,
                         dq: int = DQ_PLAIN) -> NF4Weight:
    """Q = quantize(fl32(W - L1 L2)) with the fp64 low-rank product (qlora_lq_quantize_residual)."""
    lib = load()
    N, K = W.shape
    r = L1.shape[1]
    w = NF4Weight.empty(N, K, W.device, format, dq)
    ws = torch.empty(max(16, int(lib.qlora_lq_workspace_bytes(N, K, r, 0, dq))), dtype=torch.uint8, device=W.device)
    s = w.c_struct()
    _check(lib.qlora_lq_quantize_residual(_ptr(W), _ptr(L1), _ptr(L2), r, ctypes.byref(s), _ptr(ws), ws.numel(),
                                          _stream()), "qlora_lq_quantize_residual")
    return w


def lq_lowrank(W: torch.Tensor, Q: NF4Weight | None, Omega: torch.Tensor, r: int, power: int = 2):
    """(L1 [N, r], L2 [r, K]) ~ rank-r part of W - W'(Q) (of W when Q is None) (qlora_lq_lowrank)."""
    lib = load()
    N, K = W.shape
    l = Omega.shape[1]
    L1 = torch.empty((N, r), dtype=torch.float32, device=W.device)
    L2 = torch.empty((r, K), dtype=torch.float32, device=W.device)
    dq = Q.dq if Q is not None else DQ_PLAIN
    ws = torch.empty(max(16, int(lib.qlora_lq_workspace_bytes(N, K, r, l, dq))), dtype=torch.uint8, device=W.device)
    s = Q.c_struct() if Q is not None else None
    _check(lib.qlora_lq_lowrank(_ptr(W), N, K, ctypes.byref(s) if s is not None else None, _ptr(Omega), l, power, r,
                                _ptr(L1), _ptr(L2), _ptr(ws), ws.numel(), _stream()), "qlora_lq_lowrank")
    return L1, L2


def dequantize(w: NF4Weight, out: torch.Tensor | None = None) -> torch.Tensor:
    lib = load()
    if out is None:
        out = torch.empty((w.rows, w.cols), dtype=torch.bfloat16, device=w.codes.device)
    s = w.c_struct()
    _check(lib.qlora_dequantize(ctypes.byref(s), _ptr(out), _stream()), "qlora_dequantize")
    return out


def linear_fwd(w: NF4Weight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float, save_h: bool = True,
               out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
               h_out: torch.Tensor | None = None):
    """Y = X W'^T + s (X A^T) B^T.  Returns (Y bf16 [M,N], H fp32 [M,r] or None)."""
    lib = load()
    M, r = X.shape[0], A.shape[0]
    Y = out if out is not None else torch.empty((M, w.rows), dtype=torch.bfloat16, device=X.device)
    H = h_out if h_out is not None else (
        torch.empty((M, r), dtype=torch.float32, device=X.device) if save_h else None)
    need = lib.qlora_workspace_bytes(QLORA_OP_FWD, M, w.rows, w.cols, r)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=X.device)
    st = w.c_struct()
    _check(lib.qlora_linear_fwd(ctypes.byref(st), _ptr(X), M, _ptr(A), _ptr(B), r, s, _ptr(Y), _ptr(H), _ptr(ws),
                                ws.numel(), _stream()), "qlora_linear_fwd")
    return Y, H


def linear_fwd_dense(W: torch.Tensor, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                     save_h: bool = True):
    """The forward on a dense bf16 base W [N, K] from any quantizer (qlora_linear_fwd_dense)."""
    lib = load()
    N, K = W.shape
    M, r = X.shape[0], A.shape[0]
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    H = torch.empty((M, r), dtype=torch.float32, device=X.device) if save_h else None
    ws = torch.empty(lib.qlora_workspace_bytes(QLORA_OP_FWD_DENSE, M, N, K, r), dtype=torch.uint8, device=X.device)
    _check(lib.qlora_linear_fwd_dense(_ptr(W), N, K, _ptr(X), M, _ptr(A), _ptr(B), r, s, _ptr(Y), _ptr(H), _ptr(ws),
                                      ws.numel(), _stream()), "qlora_linear_fwd_dense")
    return Y, H


def linear_bwd_dense(W: torch.Tensor, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
                     H: torch.Tensor | None = None):
    """The backward on a dense bf16 base W [N, K] (qlora_linear_bwd_dense): (dX, dA, dB)."""
    lib = load()
    N, K = W.shape
    M, r = X.shape[0], A.shape[0]
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=X.device)
    dA = torch.empty((r, K), dtype=torch.float32, device=X.device)
    dB = torch.empty((N, r), dtype=torch.float32, device=X.device)
    ws = torch.empty(lib.qlora_workspace_bytes(QLORA_OP_BWD_DENSE, M, N, K, r), dtype=torch.uint8, device=X.device)
    _check(lib.qlora_linear_bwd_dense(_ptr(W), N, K, _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), r, s, _ptr(H), _ptr(dX),
                                      _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream()), "qlora_linear_bwd_dense")
    return dX, dA, dB


def linear_fwd_materialized(materialize, N: int, K: int, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                            s: float, save_h: bool = True):
    """The forward with the base produced by `materialize(W_out)` (a callable that fills a bf16 CUDA
    tensor [N, K] on the current stream) through qlora_linear_fwd_materialized."""
    lib = load()
    M, r = X.shape[0], A.shape[0]
    scratch = torch.empty((N, K), dtype=torch.bfloat16, device=X.device)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    H = torch.empty((M, r), dtype=torch.float32, device=X.device) if save_h else None
    ws = torch.empty(lib.qlora_workspace_bytes(QLORA_OP_FWD_DENSE, M, N, K, r), dtype=torch.uint8, device=X.device)

    def cb(ctx, w_out, n, k, stream):
        if w_out != scratch.data_ptr() or (n, k) != (N, K):
            return 1
        materialize(scratch)
        return 0
    fn = MATERIALIZE_FN(cb)
    _check(lib.qlora_linear_fwd_materialized(fn, None, _ptr(scratch), N, K, _ptr(X), M, _ptr(A), _ptr(B), r, s,
                                             _ptr(Y), _ptr(H), _ptr(ws), ws.numel(), _stream()),
           "qlora_linear_fwd_materialized")
    return Y, H


def linear_bwd(w: NF4Weight, X: torch.Tensor, dY: torch.Tensor, A: torch.Tensor, B: torch.Tensor, s: float,
               H: torch.Tensor | None = None, outs=None, workspace: torch.Tensor | None = None):
    """Returns (dX bf16 [M,K], dA fp32 [r,K], dB fp32 [N,r]); the frozen W' gets no gradient."""
    lib = load()
    M, r = X.shape[0], A.shape[0]
    if outs is None:
        dX = torch.empty((M, w.cols), dtype=torch.bfloat16, device=X.device)
        dA = torch.empty((r, w.cols), dtype=torch.float32, device=X.device)
        dB = torch.empty((w.rows, r), dtype=torch.float32, device=X.device)
    else:
        dX, dA, dB = outs
    need = lib.qlora_workspace_bytes(QLORA_OP_BWD, M, w.rows, w.cols, r)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=X.device)
    st = w.c_struct()
    _check(lib.qlora_linear_bwd(ctypes.byref(st), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B), r, s, _ptr(H), _ptr(dX),
                                _ptr(dA), _ptr(dB), _ptr(ws), ws.numel(), _stream()), "qlora_linear_bwd")
    return dX, dA, dB
