import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 GPU (runs the CUDA path)")


@pytest.fixture(scope="session", autouse=True)
def _built():
    """Build the oracle (gcc) and the CUDA library (nvcc) if they are stale."""
    import oracle

    oracle.build()
    from sliding_window_attention_fwd_b200 import build as swa_build

    swa_build.build()
    yield


def has_gpu() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False
