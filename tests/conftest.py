import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def hcl():
    """The CUDA library; GPU tests skip without a device and fail loudly without libhcl.so."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from heavily_compressed_long_b200 import api, _lib
    _lib.lib()  # raises if libhcl.so is missing
    return api
