import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity runs")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def spin_gpu():
    """The CUDA library on a B200. Fails (does not skip) when CUDA is absent, so
    a GPU run can never pass on a fallback."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from online_hadamard_rotation_b200 import build
    build.build()
    import online_hadamard_rotation_b200 as spin
    spin.lib()
    return spin
