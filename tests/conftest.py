import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    return oracle.lib()


def cuda_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def gpu():
    """The product library on cuda:0. Fails (never falls back) if the library is missing."""
    if not cuda_available():
        pytest.skip("no CUDA device")
    import nvfp4_block_scaled_13_b200 as nv

    nv.load()   # raises if the shared library is absent
    return nv
