import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: CPU test that takes more than a few seconds")


@pytest.fixture(scope="session")
def cuda_lib():
    """The C-ABI library, loaded on a GPU machine (the product path fails loudly without it)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sequence_exact_attention_ring_b200 import binding
    return binding.load()
