import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload parity (minutes)")


@pytest.fixture(scope="session")
def oracle():
    import oracle as _o
    _o.build()
    return _o


@pytest.fixture(scope="session")
def moe():
    """The product binding; on a machine with a GPU it must load the CUDA library."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import mixture_experts_layer_aux_b200 as m
    m.load()
    return m
