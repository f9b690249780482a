import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (runs the sm_100a kernels through the C ABI)")
    config.addinivalue_line("markers", "slow: long CPU or GPU run (full-size model)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.lib()


@pytest.fixture(scope="session")
def i4lib():
    """The built CUDA library (built in-tree on first use when missing or stale)."""
    from int4_weight_only_02_b200 import build as b
    b.build()
    import int4_weight_only_02_b200 as i4
    return i4


@pytest.fixture(scope="session")
def cuda(i4lib):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("a CUDA device is required for -m gpu tests")
    torch.cuda.init()
    return torch.device("cuda:0")

