import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def lib():
    """The C-ABI library (loads on CPU; compute calls need a GPU)."""
    from aurora_orthogonalised_optimizer_b200 import _abi
    return _abi.load()


@pytest.fixture(autouse=True)
def _checked_build_status(request):
    """Under the bounds-checked library (AURORA_MUON_CHECKED=1) every GPU test
    must also leave no failed index test behind."""
    yield
    if os.environ.get("AURORA_MUON_CHECKED") == "1" and request.node.get_closest_marker("gpu"):
        from aurora_orthogonalised_optimizer_b200 import _abi as A
        st = A.last_device_status()
        assert st == A.MUON_OK, (A.status_string(st), "line", A.last_check_line())
