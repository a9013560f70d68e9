"""The debug-bounds build (libexl3_debug.so, compiled with -DEXL3_DEBUG_BOUNDS):
its kernels check every access of the product paths to the packed words, the
workspace and the outputs, and would report a failed check as EXL3_ERR_BOUNDS
through exl3_workspace_status (skipping the access, never trapping).  Small
in-range cases of every product path run through it in a fresh process; they
must match the oracle with every status word clean."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def test_debug_bounds_build_in_range_cases_clean():
    lib = os.path.join(ROOT, "gemm_exl3_gemv_b200", "libexl3_debug.so")
    assert os.path.exists(lib), "build the library first (python -m gemm_exl3_gemv_b200.build)"
    env = dict(os.environ, EXL3_LIBRARY=lib)
    out = subprocess.run([sys.executable, os.path.join(HERE, "debug_bounds_cases.py")], cwd=ROOT, env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stdout[-2000:] + out.stderr[-3000:]
    assert "debug-bounds cases ok" in out.stdout
