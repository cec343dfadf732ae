import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_lib():
    """The built C-ABI library, loaded through the binding (GPU tests only)."""
    if not _has_gpu():
        pytest.skip("no CUDA device")
    from nvfp4_bit_precision_quantize_b200 import binding, build
    build.build()
    binding.load()
    return binding
