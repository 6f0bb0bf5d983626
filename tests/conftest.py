import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    """Build the in-tree library when it is missing (a fresh checkout); a failed build leaves
    it missing, so the tests that load it still fail loudly."""
    lib = os.path.join(ROOT, "diffusion_transformer_denoiser_dit_b200", "libdit_b200.so")
    if not os.path.exists(lib):
        from diffusion_transformer_denoiser_dit_b200 import build as b
        try:
            b.build()
        except Exception as e:  # reported by the tests that need the library
            sys.stderr.write(f"building libdit_b200.so failed: {e}\n")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long-running CPU work (full-size oracle samples)")


@pytest.fixture(scope="session")
def lib():
    """The built CUDA library on a GPU machine (fails loudly if it is missing)."""
    from diffusion_transformer_denoiser_dit_b200 import binding
    return binding.load()
