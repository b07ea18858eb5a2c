import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes of CPU oracle time)")


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test selected but torch.cuda.is_available() is False")
    return torch.device("cuda:0")


def pytest_terminal_summary(terminalreporter):
    from tests._helpers import MARGINS
    if MARGINS:
        terminalreporter.write_sep("-", "parity margins (max|err| / max|ref|; tolerance 2e-2 bf16, 1e-4 fp32)")
        for name, text in MARGINS:
            terminalreporter.write_line(f"{name}: {text}")
