"""The debug build (libgdr2_debug.so, compiled with -DGDR2_DEBUG) on a B200: its kernels check their chunk,
chain, tile, TMEM-map and output indices and report a failed check through gdr2_check as GDR2_ERR_BOUNDS
(no trap). tests/debug_build_driver.py runs one small case per kernel family (per-chain, chunk-parallel, the
chunk-level scan, packed batches with and without grouped value heads, decode) in a child process that loads
the debug library, and checks both that no index check failed and that the outputs agree with the oracle.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_index_checks_pass():
    env = dict(os.environ, GDR2_DEBUG_BUILD="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_build_driver.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    assert "debug build: all cases ok" in r.stdout
