import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA path's binding, built in-tree first if it is missing or older than its sources
    (a no-op otherwise); GPU tests fail loudly if it cannot be built or loaded."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but no CUDA device is visible")
    import __graft_entry__
    __graft_entry__._build_module().build()
    import long_sequence_attention_b200 as lsa
    return lsa


@pytest.fixture(scope="session")
def cuda_lib_host():
    """The binding for host-only calls (no GPU needed): built in-tree if missing or stale."""
    import __graft_entry__
    __graft_entry__._build_module().build()
    import long_sequence_attention_b200 as lsa
    return lsa
