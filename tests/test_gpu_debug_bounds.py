"""The bounds-checked build: every kernel compiled with -DFA_DEBUG_BOUNDS,
whose index checks record FA_ERR_BOUNDS in the device status word and skip
the access instead of touching memory outside a buffer.  It stands in for a
memory checker: the build runs small cases of every kernel (dense forward and
backward in both dQ modes, GQA, windows, softcap, packed batches, qkvpacked
views, ALiBi, E4M3, paged and contiguous decode with every box size and the
cp.async fallback, rotary) with a clean status word and oracle parity.  The
cases run in a child process (tests/_bounds_child.py), since a process loads
one copy of the library."""

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


def test_bounds_checked_build_runs_clean():
    from exact_attention_121_b200 import build
    lib = build.build(debug_bounds=True)
    assert os.path.basename(lib) == "libfa_debug.so"
    r = subprocess.run([sys.executable, os.path.join(HERE, "_bounds_child.py")], capture_output=True, text=True,
                       timeout=900)
    assert r.returncode == 0, (r.stdout[-3000:] + r.stderr[-3000:])
    assert "bounds-checked build clean" in r.stdout
