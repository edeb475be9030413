import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def cuda_lib():
    """The built CUDA library (tests that need a GPU only)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from xlstm_mlstm_cell_b200 import binding
    return binding.load()
