import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built library")


def gpu_available() -> bool:
    try:
        import torch

        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.fixture(scope="session")
def cuda_device():
    if not gpu_available():
        pytest.skip("no CUDA device")
    import torch

    return torch.device("cuda:0")


def pytest_sessionfinish(session, exitstatus):
    """Writes the parity margins the GPU tests recorded (see margins.py) to stderr."""
    try:
        from margins import summary_lines
    except ImportError:
        return
    lines = summary_lines()
    if lines:
        sys.stderr.write("\n" + "\n".join(lines) + "\n")
        sys.stderr.flush()
