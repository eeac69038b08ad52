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
def oracle_mod():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def librq_built():
    """Builds (if stale) and loads the in-tree librq.so; GPU tests need a device."""
    import torch
    from residual_bit_kv_b200 import build
    build.build()
    import residual_bit_kv_b200.librq as L
    L.load()
    return L


@pytest.fixture(scope="session")
def cuda_dev(librq_built):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    torch.cuda.init()
    return torch.device("cuda")
