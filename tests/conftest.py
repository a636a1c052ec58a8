import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session", autouse=True)
def built_libraries():
    """The CUDA library (and its test-hook build) and the CPU oracle, compiled
    in-tree; each build is skipped when it is newer than its sources."""
    import dense_fp8_gemm_b200.build as b
    import oracle.build as ob
    b.build()
    b.build_test_hooks()
    ob.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
