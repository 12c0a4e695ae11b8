import os
import shutil
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _oracle
    _oracle.build()
    return _oracle


@pytest.fixture
def work_dir():
    """A scratch directory inside the repository's ignored _build/ folder,
    removed after the test."""
    base = os.path.join(ROOT, "_build", "tests")
    os.makedirs(base, exist_ok=True)
    d = tempfile.mkdtemp(dir=base)
    yield d
    shutil.rmtree(d, ignore_errors=True)
