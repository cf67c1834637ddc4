"""The library's debug variant (libradattn_debug.so, built with -DRA_DEBUG_BOUNDS):
its kernels check every global index and TMA coordinate they derive from their
inputs (the dispatch order, the block-CSR rows and column indices) and record a
failure in the device error word instead of making the access.  Its self-test
must report a planted failing check (on an index it never uses); the small
parity cases, forward and backward in both modes, and a streaming SWC run must
pass through it with no check firing.  Runs in a child process, because the
variant is chosen when the binding is imported."""
import os
import subprocess
import sys

import pytest

from tests import _gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_library_checks_and_passes_the_small_cases():
    _gpu.need_gpu()
    # build (or bring up to date) the debug variant; a no-op when it is current
    subprocess.run([sys.executable, os.path.join(ROOT, "static_sparse_attention_b200", "build.py"), "--debug"],
                   check=True, capture_output=True, timeout=900)
    env = dict(os.environ, RA_LIBRARY_VARIANT="debug")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "_debug_bounds_run.py")], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "debug bounds ok" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
