"""Outputs stay inside their buffers: every output of the quantizer, the
dequantizer, the few-token forward and the tensor-core linear (forward and
backward) is written into a view with 4 KB of canary bytes on both sides,
which must be unchanged afterwards (tests/canary_cases.py; the memory checker
that would do this is not available here)."""

import pytest

pytestmark = pytest.mark.gpu


def test_outputs_stay_inside_their_buffers(lib):
    from tests import canary_cases
    out = canary_cases.run_all()
    assert len(out) > 20
