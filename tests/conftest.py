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


@pytest.fixture(scope="session")
def rfb_lib():
    """The CUDA library, built in-tree if its sources are newer than the .so."""
    from rank_biased_window_b200 import build as b
    b.build()
    import rank_biased_window_b200 as rfb
    rfb.load_library()
    return rfb


@pytest.fixture(scope="session")
def cuda_dev(rfb_lib):
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    return torch.device("cuda", 0)
