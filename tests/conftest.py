import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: long CPU or GPU case")


@pytest.fixture(scope="session")
def cuda_ok():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return True


# GPU tests run the library in debug mode: every call synchronises and reports
# device-side bounded-wait failures as LORA_ERR_TIMEOUT instead of silent garbage.
os.environ.setdefault("LORA_MLP_DEBUG", "1")
os.environ.setdefault("LORA_MLP_WAIT_LIMIT_MS", "3000")
