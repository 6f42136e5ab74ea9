"""The boundary as a C client sees it: tests/c_abi_check.c includes
include/qlora.h, is compiled as C99 (-pedantic -Werror) and as C++17, links
against libqlora.so and calls the host side of the ABI (no GPU needed).  What
it prints must agree with the oracle (the code tables, the storage sizes) and
with the Python binding (workspace sizes, status strings)."""

import os
import shutil
import subprocess

import numpy as np
import pytest

import bit_quantized_lora_nf4_b200 as q
from oracle import nf4 as onf4

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi_check.c")
INCLUDE = os.path.join(ROOT, "include")
PKG = os.path.dirname(q.LIB_PATH)


def _build_and_run(tmp_path, compiler, std):
    if shutil.which(compiler) is None:
        pytest.skip(f"{compiler} not installed")
    if not os.path.exists(q.LIB_PATH):
        pytest.skip("libqlora.so not built")
    exe = str(tmp_path / f"c_abi_{compiler}")
    lang = ["-x", "c++"] if compiler == "g++" else []
    cmd = [compiler, *lang, std, "-pedantic", "-Wall", "-Wextra", "-Werror", "-I", INCLUDE, SRC,
           "-x", "none", "-L", PKG, "-lqlora", f"-Wl,-rpath,{PKG}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    return {k: v for k, v in (line.split(" ", 1) for line in r.stdout.splitlines())}


def _floats(hexwords):
    return np.array([int(h, 16) for h in hexwords.split()], dtype=np.uint32).view(np.float32)


@pytest.mark.parametrize("compiler,std", [("gcc", "-std=c99"), ("g++", "-std=c++17")])
def test_c_client(tmp_path, compiler, std):
    out = _build_and_run(tmp_path, compiler, std)
    assert np.array_equal(_floats(out["nf4"]).view(np.uint32), onf4.nf4_codebook().view(np.uint32))
    for fid, name in ((0, "nf4"), (1, "fp4"), (2, "int4")):
        lv = _floats(out[f"levels{fid}"])
        th = _floats(out[f"thresh{fid}"])
        assert np.array_equal(lv.view(np.uint32), onf4.codebook(name).view(np.uint32)), name
        # each threshold is the largest fp32 that still takes the lower of two
        # distinct neighbouring levels, by the oracle's nearest-level rule
        for i in range(15):
            if lv[i] == lv[i + 1]:
                continue
            at = np.array([th[i]], dtype=np.float32)
            above = np.nextafter(at, np.float32(np.inf))
            assert onf4.nearest_code(at, lv)[0] <= i, (name, i)
            assert onf4.nearest_code(above, lv)[0] >= i + 1, (name, i)
    assert int(out["bad_format"]) == 1 and int(out["null_levels"]) == 1 and int(out["null_codebook"]) == 1
    codes, absmax, gs, gs_signed = (int(v) for v in out["sizes"].split())
    n = 4096 * 11008
    assert codes == n // 2 and absmax == onf4.num_blocks(n) and gs == 4 * onf4.num_groups(n)
    assert gs_signed == gs + 4
    ws_f, ws_b, ws_min = (int(v) for v in out["ws"].split())
    assert ws_f == q.workspace_bytes(q.QLORA_OP_FWD, 4096, 11008, 4096, 64)
    assert ws_b == q.workspace_bytes(q.QLORA_OP_BWD, 4096, 11008, 4096, 64)
    assert 0 < ws_min <= ws_f
    ok, bad = out["status"].split("|")
    assert ok == q.STATUS_NAMES[0] and bad == q.STATUS_NAMES[1]
