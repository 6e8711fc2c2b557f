import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libzmoe")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


_BUILT = []


@pytest.fixture(autouse=True)
def _ensure_libzmoe_for_gpu_tests(request):
    """GPU tests use the in-tree libzmoe.so; build it once (incrementally) if needed."""
    if request.node.get_closest_marker("gpu") is not None and not _BUILT:
        from sparse_moe_decoder_b200 import build as B
        B.build()
        _BUILT.append(True)
    yield
