import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU test")


@pytest.fixture(scope="session")
def host_gen():
    import workload
    workload.build_host()
    return workload


@pytest.fixture(scope="session")
def csa2_lib():
    """The built CSA2 library (nvcc for sm_100a; a few seconds) and its binding."""
    from fp4_kv_cache_decode_b200 import _build, csa2
    _build.build()
    return csa2
