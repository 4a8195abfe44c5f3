import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _o
    return _o.get()


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library; GPU tests fail loudly (not skip) if it cannot be loaded."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test selected but no CUDA device is visible")
    from mamba_ssd_scan_02_b200 import ssd
    ssd.load()
    return ssd
