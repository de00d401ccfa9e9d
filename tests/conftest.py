import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


GOLDEN = os.path.join(ROOT, "tests", "golden")


def read_golden(name):
    """Rows of a whitespace-separated golden fixture, comments stripped."""
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                rows.append(line.split())
    return rows


@pytest.fixture(scope="session")
def golden():
    return read_golden


@pytest.fixture(params=["cpp", "numpy"], scope="session")
def impl(request):
    """Each statement of the oracle in turn: the C++ one (the oracle the GPU
    tests use) and the numpy one. Every pin must hold for both."""
    import oracle
    return oracle.cpp_oracle if request.param == "cpp" else oracle.numpy_oracle
