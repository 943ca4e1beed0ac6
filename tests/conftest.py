import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size configuration (minutes)")


def pytest_collection_modifyitems(config, items):
    # a gpu-marked test on a machine without a GPU is a collection error of intent:
    # skip it with a clear reason rather than letting the library raise
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_sessionfinish(session, exitstatus):
    # Under the bounds-checked library (DIFFATTN_EXPECT_NO_VIOLATIONS=1, set by
    # tests/test_gpu_bounds_checked.py for its child run), every kernel access must have
    # stayed inside its tensor: a non-zero count fails the session.
    if os.environ.get("DIFFATTN_EXPECT_NO_VIOLATIONS") != "1":
        return
    import differential_attention_05_b200 as da
    n = da.diffattn_debug_bounds_violations()
    print(f"\nbounds-checked library: {n} out-of-range accesses skipped")
    if n is None or n != 0:
        session.exitstatus = 1
