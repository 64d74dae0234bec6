import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")


@pytest.fixture(scope="session")
def lib():
    """The CUDA library through its Python binding (GPU tests only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    from sparse_int4_linear_b200 import slim
    return slim


@pytest.fixture
def tune(lib, monkeypatch):
    """Set SLIM_* tuning variables for one test.  The library reads them once,
    so it is told to re-read them after every change and after the test."""
    def set_vars(**kv):
        for k, v in kv.items():
            monkeypatch.setenv(k, v)
        lib.tuning_reload()
    yield set_vars
    monkeypatch.undo()
    lib.tuning_reload()
