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
    """The CUDA library through its Python binding; fails loudly when the
    extension is missing (there is no CPU fallback)."""
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import shared_kv_decoder_b200 as yoco
    yoco.load()
    return yoco
