import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle


@pytest.fixture(scope="session")
def syn():
    import synth
    synth._load()
    return synth


@pytest.fixture(scope="session")
def kvq():
    """The C-ABI library's Python binding, built in-tree if missing (nvcc)."""
    from bit_kv_cache_18_b200 import build
    import bit_kv_cache_18_b200 as m
    if not os.path.exists(m.LIB_PATH):
        build.build()
    m.lib()
    return m


@pytest.fixture(scope="session")
def cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
