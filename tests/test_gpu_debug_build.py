"""The bounds-checked debug build on the GPU: tests/_debug_cases.py runs in a child process with
QLORA_LIBRARY=debug, so every kernel checks its TMA start coordinates, partial-sum pieces and
segments, arrival counters and output rows before it touches memory.  Every case must leave the
status word clean (no check fired) and match the oracle."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_debug_build_small_ragged_cases():
    from bit_quantized_base_b200 import build
    build.build(debug=True)
    env = dict(os.environ, QLORA_LIBRARY="debug", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, os.path.join(HERE, "_debug_cases.py")], cwd=ROOT,
                         env=env, capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stdout[-3000:] + out.stderr[-3000:]
    assert "all debug-build cases passed" in out.stdout
