"""The GPU parity suites run once more against the bounds-checked library.

In libdiffattn_debug.so (built with DIFFATTN_DEBUG) every raw global-memory access of the
kernels -- the epilogue stores, the statistics, the decode's copies, workspace records and
block-table reads, the fp32 kernels' rows -- is checked against the extent of its tensor as
computed on the host from the shapes and strides; an access outside it is skipped, reported
through the status word and counted, and nothing traps. (It stands in for a memory checker,
which this pool does not offer.) The child pytest run below takes the ragged, empty,
chunked, windowed, packed, paged and full-size cases of those suites, compares every result
with the float64 oracle as the normal run does, and fails if any access was skipped
(tests/conftest.py reads the counter at the end of the session).
"""
import os
import subprocess
import sys

import pytest

from differential_attention_05_b200 import build as B

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SUITES = ["test_gpu_prefill_bf16.py", "test_gpu_chunked_window.py", "test_gpu_varlen_prefill.py",
          "test_gpu_paged_decode.py", "test_gpu_decode_v1.py", "test_gpu_lambda_simt_decode.py",
          "test_gpu_backward.py"]


def test_parity_suites_under_the_bounds_checked_library():
    lib = B.LIB_DEBUG
    assert os.path.exists(lib), "libdiffattn_debug.so is missing: python -m differential_attention_05_b200.build --debug"
    env = dict(os.environ, DIFFATTN_LIBRARY=lib, DIFFATTN_EXPECT_NO_VIOLATIONS="1")
    cmd = [sys.executable, "-m", "pytest", "-q", "-x", "-m", "gpu", "-p", "no:cacheprovider",
           *[os.path.join(HERE, f) for f in SUITES]]
    r = subprocess.run(cmd, env=env, capture_output=True, text=True, timeout=1800)
    tail = (r.stdout + r.stderr)[-3000:]
    assert r.returncode == 0, tail
    assert "0 out-of-range accesses skipped" in r.stdout, tail
