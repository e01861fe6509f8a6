import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_native():
    """Build the CUDA library (nvcc, sm_100a) if missing or stale, so the
    tests always run the real native path."""
    import runpy
    runpy.run_path(os.path.join(ROOT, "streaming_top_b200", "build.py"))["build"]()


_build_native()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running (large workloads)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.load()
