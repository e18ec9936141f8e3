import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes)")


@pytest.fixture(scope="session")
def cuda_dev():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test collected without a CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(params=["numpy", "cpp"])
def O(request):
    """The oracle under test: the numpy one (oracle/moe_oracle.py) or the
    single-threaded C++ one (oracle/moe_oracle_ref.cpp).  Every pin that
    takes this fixture runs against both."""
    if request.param == "numpy":
        from oracle import moe_oracle as m
    else:
        from oracle import cpp_oracle as m
    return m
