import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(autouse=True)
def _guard_bands(request):
    """After every GPU test: the guard bands around each device buffer the test handed
    the library (tests/gpu_cases.py) must be intact."""
    yield
    if request.node.get_closest_marker("gpu") is None:
        return
    mod = sys.modules.get("tests.gpu_cases")
    if mod is not None:
        mod.check_guards()
