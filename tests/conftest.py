import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload (seconds to minutes)")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


def pytest_sessionfinish(session, exitstatus):
    # Under the bounds-checked library (MOE_LIBRARY=libmoe_check.so), write the
    # device's bounds-check failure count and first failing line to the file
    # MOE_BOUNDS_REPORT names (test_gpu_check_bounds.py reads it).
    path = os.environ.get("MOE_BOUNDS_REPORT")
    if not path:
        return
    import combine_moe_route_13_b200 as M
    n, line = M.moe_debug_bounds_failures()
    with open(path, "w") as f:
        f.write(f"{n} {line}\n")
