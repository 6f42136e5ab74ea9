"""The debug build (libqlora_debug.so, QLORA_BOUNDS_CHECK): every global-memory
index of the quantizer, the dequantizer and the few-token forward is checked
against its buffer, and a miss latches QLORA_ERR_BOUNDS instead of trapping.
The canary cases run on it in a child process (QLORA_DEBUG_BOUNDS=1 selects the
library): no bounds error, canaries intact, and outputs bit-identical to the
release build's."""

import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_checks_pass_and_match_the_release_build(lib, tmp_path):
    from tests import canary_cases
    release = canary_cases.run_all()
    out = tmp_path / "debug.npz"
    env = dict(os.environ, QLORA_DEBUG_BOUNDS="1")
    r = subprocess.run([sys.executable, "-m", "tests.canary_cases", str(out)], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    d = np.load(out)
    assert str(d["library"]) == "libqlora_debug.so"
    for k, v in release.items():
        assert np.array_equal(d[k], v), k
