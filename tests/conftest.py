import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (full-size workloads)")


def read_golden(name):
    """Golden fixture -> (params dict, data lines); '#' lines are comments."""
    params, lines = {}, []
    with open(os.path.join(GOLDEN, name)) as f:
        for raw in f:
            s = raw.strip()
            if not s or s.startswith("#"):
                continue
            parts = s.split()
            if parts[0][0].isalpha():
                # "key value" or "key v1 v2 ..." (a list of numbers)
                params[parts[0]] = parts[1] if len(parts) == 2 else [float(x) for x in parts[1:]]
            else:
                lines.append(s)
    return params, lines


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(scope="session")
def duo():
    """The ctypes binding; builds libduo.so first when it is missing or stale."""
    from head_split_kv_b200 import build as B
    B.build()
    from head_split_kv_b200 import duo as D
    return D
