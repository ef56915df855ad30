"""The debug-bounds build: the library compiled with -DTTT_DEBUG_BOUNDS
(libttt_b200_dbg.so), whose kernels check their index arithmetic (row,
column and batch ranges of the global stores, TMA x coordinates on 16-byte
boundaries, boxes inside their shared-memory slots, slabs inside their
matrices) and record TTT_ERR_BOUNDS instead of making the access. It stands in
for a memory checker, which cannot run on these GPUs.

The hot path's parity tests run again in a child process that loads the
checked library; their helpers assert a clean device status after every call.
"""
import os
import subprocess
import sys

import pytest

from linear_attention_ttt_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PARITY = ["tests/test_parity_linear_gpu.py", "tests/test_parity_lact_gpu.py",
          "tests/test_parity_lact_momentum_gpu.py", "tests/test_cp_gpu.py",
          "tests/test_zz_no_alloc.py", "tests/test_debug_bounds_gpu.py"]
IN_CHILD = os.environ.get("TTT_B200_LIB", "").endswith("_dbg.so")


@pytest.mark.gpu
def test_bounds_failure_is_reported_without_a_fault():
    """A failed check is recorded as TTT_ERR_BOUNDS and the context stays usable
    (debug build); the normal build has no checks and says so."""
    lib = ops.load()
    code = lib.ttt_selftest_bounds(None)
    if not IN_CHILD:
        assert code == ops.ERR_CODES["TTT_ERR_UNSUPPORTED"]
        return
    assert code == 0
    assert ops.device_status() == ops.ERR_CODES["TTT_ERR_BOUNDS"]
    assert ops.device_status() == 0  # reading it cleared it


@pytest.mark.gpu
@pytest.mark.skipif(IN_CHILD, reason="this is the parent test")
def test_hot_path_parity_under_the_debug_bounds_build():
    path = build.build(debug_bounds=True)
    env = dict(os.environ, TTT_B200_LIB=path)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu",
                        "-p", "no:cacheprovider", *PARITY],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=1800)
    assert r.returncode == 0, r.stdout[-4000:] + r.stderr[-2000:]
    assert " passed" in r.stdout, r.stdout[-1000:]
