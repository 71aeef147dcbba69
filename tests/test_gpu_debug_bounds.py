"""The bounds-checking debug build (-DWINATTN_DEBUG): every token index the
kernels form and every TMA box origin is checked against the map, and a
violation is reported through the device status word
(WINATTN_ERR_DEVICE_BOUNDS) with the access clamped into the map, never a
trap.  Here that build runs the small whole-map parity cases (every kernel;
shifted, odd-shifted and padded grids; packed and ragged tiles), the saved
log-sum-exp, the backward, the gated residual and the RIB/CLA pieces in a
child process; each of those tests asserts a clean status word, so any
out-of-range index fails them."""
import os
import subprocess
import sys

import pytest

from windowed_attention_vision_b200 import _lib

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_debug_build_finds_no_out_of_range_index():
    assert os.path.exists(_lib.DEBUG_LIB_PATH), "build the debug library first (build.build(debug=True))"
    env = dict(os.environ, WINATTN_LIB=_lib.DEBUG_LIB_PATH)
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           "tests/test_gpu_parity.py", "tests/test_gpu_backward.py", "tests/test_gpu_sparse.py",
           "tests/test_gpu_rib_cla.py", "tests/test_gpu_rescale.py",
           "-k", "small_full or tiny or lse or backward or gated or rib or cla or rescale"]
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
    tail = "\n".join((r.stdout + r.stderr).strip().splitlines()[-15:])
    assert r.returncode == 0 and " passed" in r.stdout, tail
