import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU work (full-size oracle samples)")


@pytest.fixture(scope="session")
def lib():
    """The built CUDA library on a GPU machine (fails loudly if it is missing)."""
    from diffusion_transformer_denoiser_dit_b200 import binding
    return binding.load()
