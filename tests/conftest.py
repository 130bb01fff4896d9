import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def cuda_lib():
    """The CUDA library through its C ABI; the test fails loudly if it is missing."""
    import torch

    if not torch.cuda.is_available():
        pytest.fail("gpu test collected without a CUDA device")
    from mla_flash_attention_attn_b200 import binding

    return binding.load()
