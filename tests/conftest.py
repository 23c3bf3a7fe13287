import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size workload")


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def kvc():
    """The C-ABI binding on a CUDA device; the library must exist (no fallback)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from fp4_compressed_kv_b200 import build, kvc as binding
    build.build()
    binding.lib()
    return binding
