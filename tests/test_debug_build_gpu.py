"""The bounds-checked build (compiled with -DFA_DEBUG: every TMA coordinate,
TMEM column range and directly indexed global address checked before use).

On small and ragged shapes (N in {1, 129, 300}, d in {64, 128}, causal and
full) through every entry point, no check may fire (the device error word
stays clean) and every result must match the float64 oracle at the stated
tolerances.  The debug library runs in a child process (FA_LIBRARY selects
it) so that it never mixes with the release library of this process.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))


def test_debug_build_small_and_ragged_shapes():
    from exact_attention_117_b200 import build
    lib = build.build(debug=True)
    env = dict(os.environ, FA_LIBRARY=lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_build_check.py")], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert "cases clean" in r.stdout
