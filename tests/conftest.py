import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def _ensure_built():
    import synth
    import oracle
    if not (os.path.exists(synth.HOST_SO) and os.path.exists(synth.DEV_SO)):
        synth.build()
    if not os.path.exists(oracle.SO):
        oracle.build()


_ensure_built()


def has_gpu() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def gpu():
    if not has_gpu():
        pytest.fail("GPU test selected but no CUDA device is visible")
    import torch
    return torch.device("cuda:0")
