"""Build libqlora.so in-tree with nvcc for sm_100a.

    python -m bit_quantized_lora_nf4_b200.build        (or build() from Python)

Objects go to ``_build/`` at the repository root; the shared library is
written next to this file so that the binding finds it without installation.
"""

from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
OBJDIR = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libqlora.so")

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ARCH + ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-I", INCLUDE, "-I", CSRC,
                 "-Xptxas", "-warn-spills"]
# Files whose fp32 arithmetic must match IEEE round-to-nearest step by step.
NO_FMAD = {"nf4_quant.cu", "qgemm.cu", "lora_gemm.cu", "gemv.cu", "api.cu"}


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    return sorted(f for f in os.listdir(CSRC) if f.endswith(".cu"))


DEBUG_OBJDIR = os.path.join(OBJDIR, "debug")
DEBUG_LIB = os.path.join(PKG, "libqlora_debug.so")
# The debug build: global-memory indices of the quantizer, dequantizer and
# few-token kernels checked against their buffers (QLORA_ERR_BOUNDS, no trap).
DEBUG_FLAGS = ["-DQLORA_BOUNDS_CHECK"]


def _compile(src: str, verbose: bool, debug: bool = False) -> str:
    obj = os.path.join(DEBUG_OBJDIR if debug else OBJDIR, src.replace(".cu", ".o"))
    cmd = [_nvcc()] + COMMON + (DEBUG_FLAGS if debug else []) + (["-fmad=false"] if src in NO_FMAD else []) + [
        "-c", os.path.join(CSRC, src), "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{res.stdout}\n{res.stderr}")
    if verbose:
        sys.stderr.write(res.stderr)
    return obj


def _stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(INCLUDE, f) for f in os.listdir(INCLUDE)]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Build libqlora.so (or, with debug=True, libqlora_debug.so) if a source is newer."""
    lib = DEBUG_LIB if debug else LIB
    if not force and not _stale(lib):
        return lib
    os.makedirs(DEBUG_OBJDIR if debug else OBJDIR, exist_ok=True)
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, debug), sources()))
    tmp = lib + ".tmp"
    cmd = [_nvcc()] + ARCH + ["-shared", "-o", tmp] + objs + ["-lcuda"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"link failed:\n{res.stdout}\n{res.stderr}")
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv, debug="--debug" in sys.argv))
