import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


import pytest  # noqa: E402


@pytest.fixture(scope="session")
def cuda_lib():
    """Builds (if stale) and loads the CUDA library; GPU tests fail loudly without it."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from denoiser_attention_b200 import build, binding
    build.build()
    return binding.lib()
